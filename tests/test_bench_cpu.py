"""Host-side pieces of bench.py: the kernel-source hash that keys the profiled DRAM traffic, and the
roofline peaks (measured file, else the recipe fallback)."""

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


def test_peaks_come_from_the_measured_file_else_the_recipe_fallback(monkeypatch, tmp_path):
    import json
    import os
    if os.path.exists(bench.PEAKS_FILE):
        with open(bench.PEAKS_FILE) as f:
            pk = json.load(f)
        hbm, tc, tcs, src = bench.load_peaks()
        assert src == "measured"
        assert (hbm, tc, tcs) == (pk["hbm_gbs"], pk["bf16_tflops"], pk.get("bf16_tflops_sustained", pk["bf16_tflops"]))
    # the profiling recipe's fallback: 6.65 TB/s and 1.59 PFLOP/s (burst), about 1.4 sustained
    monkeypatch.setattr(bench, "PEAKS_FILE", str(tmp_path / "absent.json"))
    assert bench.load_peaks() == (6650.0, 1590.0, 1400.0, "fallback")


def test_each_kernel_has_its_own_source_hash_and_summary():
    """The traffic figure of a workload comes from the summary of the kernel that workload runs,
    keyed on that kernel's own sources."""
    assert bench.decode_kernel_of(16, False) == "etap_pair_kernel"
    assert bench.decode_kernel_of(17, False) == "etap_duo_kernel"
    assert bench.decode_kernel_of(128, True) == "etap_pair_kernel"  # the FP8 cache keeps the pair kernel
    assert bench.kernel_source_hash(kernel="etap_pair_kernel") != bench.kernel_source_hash(kernel="etap_duo_kernel")
    assert bench.profiled_traffic("mla_decode_b16_h16_q1_L65536_contiguous", "etap_duo_kernel") is None
    assert bench.profiled_traffic("anything", "untransposed_kernel") is None
    t = bench.profiled_traffic("mla_decode_b32_h128_q1_Lunif8192to32768_paged64", "etap_duo_kernel")
    assert t is not None and 1.0 <= t / 785979648 < 1.2  # the value re-read adds up to ~10% of HBM reads

