"""The algorithmic byte and flop counts behind every roofline figure bench.py reports, pinned by
brute-force pair counting and by closed forms for the headline and causal workloads."""

from __future__ import annotations

import itertools

import pytest

from mla_decode_attention_etap_b200 import workloads as W

FLOP_PER_PAIR = 2 * (576 + 512)


def brute_pairs(seqlens, q_len, heads, causal, q_lens=None):
    """Count (query column, cache row) pairs by enumeration: token t of the q real tokens of sequence b
    is cache row L - q + t, and sees row j when j <= that row (causal) or j < L."""
    n = 0
    for b, L in enumerate(seqlens):
        q = q_len if q_lens is None else q_lens[b]
        for t, j in itertools.product(range(q), range(L)):
            if not causal or j <= L - q + t:
                n += heads
    return n


@pytest.mark.parametrize("seqlens,q_len,heads,causal,q_lens", [
    ([5, 0, 17], 1, 16, False, None),
    ([5, 2, 17], 4, 16, True, None),    # L < q_len: early tokens see nothing
    ([9, 30], 3, 128, True, None),
    ([12, 7, 40], 4, 16, True, [4, 1, 0]),   # ragged: padding tokens see no row
    ([12, 7], 2, 32, False, [2, 1]),
])
def test_flops_match_brute_force(seqlens, q_len, heads, causal, q_lens):
    got = W.algorithmic_flops(seqlens, q_len, heads, causal, q_lens)
    assert got == brute_pairs(seqlens, q_len, heads, causal, q_lens) * FLOP_PER_PAIR


def test_headline_and_causal_workload_closed_forms():
    # B=16, h=16, one token, 65536 rows: 16 * 65536 * 16 pairs; 1152 bytes per cached token
    assert W.algorithmic_flops([65536] * 16, 1, 16, False) == 16 * 65536 * 16 * FLOP_PER_PAIR
    assert W.algorithmic_kv_bytes([65536] * 16) == 16 * 65536 * 1152 == 1_207_959_552
    # q_len=4 causal at L=32768: token t sees L - 3 + t rows, 4L - 6 per head and sequence
    assert W.algorithmic_flops([32768] * 16, 4, 16, True) == (4 * 32768 - 6) * 16 * 16 * FLOP_PER_PAIR
    assert W.algorithmic_flops([32768] * 16, 4, 16, True) == 73_011_101_696


def test_fp8_bytes_count_codes_and_row_scales():
    assert W.algorithmic_kv_bytes([100, 28], fp8=True) == 128 * (576 + 4)
    assert W.algorithmic_kv_bytes([0, 0]) == 0
