"""Host-side pieces of bench.py: the kernel-source hash that keys the profiled DRAM traffic."""

import bench


def test_code_only_hash_ignores_comments_not_code():
    base = "int a = 1;  // one\n\n// a comment line\nint b = 2;\n"
    assert bench.code_only(base) == bench.code_only("int a = 1;\n// other words\nint b = 2;  // two\n")
    assert bench.code_only(base) != bench.code_only("int a = 1;\nint b = 3;\n")


def test_profiled_traffic_matches_the_current_kernel_source():
    """The committed ncu summary was taken on the kernel as it stands (else bench reports null)."""
    t = bench.profiled_traffic("mla_decode_b16_h16_q1_L65536_contiguous")
    assert t is not None
    # read traffic within a few percent of the algorithmic KV bytes of the launch
    assert 1.0 <= t / (16 * 65536 * 1152) < 1.05
