"""Pins for the FP8-cache oracle (CPU only).

The FP8 cache is a storage format: row r holds E4M3 codes and one fp32 scale,
and stands for scale[r] * e4m3(code).  The attention itself is the definition
the bf16 oracle computes (FlashMLA-ETAP technical summary, Methodology), so the
pins tie the FP8 oracle to facts that do not depend on it:

* the E4M3 decoding, through a one-row decode (O = that row's V exactly), against
  PyTorch's ``float8_e4m3fn`` conversion (a library routine) for all 254 finite codes;
* with power-of-two scales every widened value is a bf16 number, so the FP8 oracle
  must equal the (already pinned) bf16 oracle on those bf16 values;
* the per-row scale: multiplying a row's scale by c multiplies its scores by c;
  with Q = 0 (all scores equal) O is the mean of the widened V rows;
* paged == contiguous with the scale array indexed like the rows; ragged q_lens;
* the numpy form (built from the E4M3 bit layout, not the C code) agrees.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import mla_oracle as om

D_QK, D_V, PAGE = 576, 512, 64
SCALE = 1.0 / 24.0


def finite_codes(rng, shape):
    c = rng.integers(0, 256, shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] ^= 0x01  # NaN codes -> the largest finite value
    return c


def torch_e4m3(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def test_e4m3_decoding_matches_the_library_for_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert codes.size == 254
    # one cache row holds all finite codes in its V columns
    kv = np.zeros((1, 1, D_QK), dtype=np.uint8)
    kv[0, 0, :254] = codes
    sc = np.ones((1, 1), dtype=np.float32)
    q = om.f64_to_bf16_bits(np.random.default_rng(0).standard_normal((1, 1, 2, D_QK)))
    o, lse = om.mla_decode_fp8(q, kv, sc, [1], scale=SCALE)
    np.testing.assert_array_equal(o[0, 0, 0, :254], torch_e4m3(codes))
    np.testing.assert_array_equal(o[0, 0, 1, :254], torch_e4m3(codes))
    # LSE of one row is its score
    k = torch_e4m3(kv[0, 0])
    qd = om.bf16_bits_to_f64(q)[0, 0]
    np.testing.assert_allclose(lse[0, 0], SCALE * qd @ k, rtol=1e-14, atol=1e-14)
    # the numpy decoding is exact too, NaN included
    assert np.array_equal(np.nan_to_num(om.e4m3_to_f64(np.arange(256)), nan=1234.5),
                          np.nan_to_num(torch_e4m3(np.arange(256, dtype=np.uint8)), nan=1234.5))


@pytest.mark.parametrize("causal,q_len", [(False, 1), (True, 3)])
def test_power_of_two_scales_equal_the_bf16_oracle(causal, q_len):
    rng = np.random.default_rng(1)
    B, h, Lm = 3, 4, 90
    lens = [90, 33, 64]
    codes = finite_codes(rng, (B, Lm, D_QK))
    sc = np.exp2(rng.integers(-12, -3, (B, Lm))).astype(np.float32)
    widened = torch_e4m3(codes) * sc[..., None].astype(np.float64)
    bits = om.f64_to_bf16_bits(widened)
    assert np.array_equal(om.bf16_bits_to_f64(bits), widened)  # exact in bf16
    q = om.f64_to_bf16_bits(rng.standard_normal((B, q_len, h, D_QK)))
    o8, l8 = om.mla_decode_fp8(q, codes, sc, lens, scale=SCALE, causal=causal)
    ob, lb = om.mla_decode(q, bits, lens, scale=SCALE, causal=causal)
    np.testing.assert_allclose(o8, ob, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l8, lb, rtol=0, atol=1e-12)


def test_row_scale_multiplies_the_scores():
    rng = np.random.default_rng(2)
    codes = finite_codes(rng, (1, 2, D_QK))
    q = om.f64_to_bf16_bits(rng.standard_normal((1, 1, 1, D_QK)))
    qd = om.bf16_bits_to_f64(q)[0, 0, 0]
    for c in (0.5, 3.0):
        sc = np.array([[0.01, 0.01 * c]], dtype=np.float32)
        o, lse = om.mla_decode_fp8(q, codes, sc, [2], scale=SCALE)
        k = torch_e4m3(codes[0]) * sc[0][:, None].astype(np.float64)
        s = SCALE * k @ qd
        w = np.exp(s - s.max())
        np.testing.assert_allclose(lse[0, 0, 0], s.max() + math.log(w.sum()), rtol=1e-13)
        np.testing.assert_allclose(o[0, 0, 0], (w / w.sum()) @ k[:, :D_V], rtol=1e-12, atol=1e-15)


def test_zero_query_gives_the_mean_of_the_widened_rows():
    rng = np.random.default_rng(3)
    L = 37
    codes = finite_codes(rng, (1, L, D_QK))
    sc = rng.uniform(1e-3, 1e-2, (1, L)).astype(np.float32)
    q = np.zeros((1, 1, 2, D_QK), dtype=np.uint16)
    o, lse = om.mla_decode_fp8(q, codes, sc, [L], scale=SCALE)
    v = torch_e4m3(codes[0, :, :D_V]) * sc[0][:, None].astype(np.float64)
    np.testing.assert_allclose(o[0, 0, 0], v.mean(axis=0), rtol=1e-12, atol=1e-16)
    np.testing.assert_allclose(lse[0, 0], math.log(L), rtol=1e-14)


def test_paged_equals_contiguous_and_numpy_agrees():
    rng = np.random.default_rng(4)
    B, h, q_len = 3, 8, 2
    lens = [130, 1, 64]
    Lm = max(lens)
    codes = finite_codes(rng, (B, Lm, D_QK))
    sc = rng.uniform(1e-3, 2e-2, (B, Lm)).astype(np.float32)
    q = om.f64_to_bf16_bits(rng.standard_normal((B, q_len, h, D_QK)))
    nblk = [(L + PAGE - 1) // PAGE for L in lens]
    perm = rng.permutation(sum(nblk))
    pool = np.zeros((sum(nblk), PAGE, D_QK), dtype=np.uint8)
    pool_sc = np.zeros((sum(nblk), PAGE), dtype=np.float32)
    bt = np.full((B, max(nblk)), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        for i in range(nblk[b]):
            blk = perm[off + i]
            bt[b, i] = blk
            n = min(PAGE, Lm - i * PAGE)
            pool[blk, :n] = codes[b, i * PAGE:i * PAGE + n]
            pool_sc[blk, :n] = sc[b, i * PAGE:i * PAGE + n]
        off += nblk[b]
    for causal in (False, True):
        oc, lc = om.mla_decode_fp8(q, codes, sc, lens, scale=SCALE, causal=causal)
        op, lp = om.mla_decode_fp8(q, pool, pool_sc, lens, block_table=bt, scale=SCALE, causal=causal)
        np.testing.assert_array_equal(oc, op)
        np.testing.assert_array_equal(lc, lp)
        on, ln = om.mla_decode_fp8_numpy(q, pool, pool_sc, lens, block_table=bt, scale=SCALE, causal=causal)
        np.testing.assert_allclose(oc, on, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lc, ln, rtol=0, atol=1e-12)


def test_ragged_fp8_matches_each_sequence_alone():
    rng = np.random.default_rng(5)
    B, h, q_len = 3, 4, 4
    lens = [50, 7, 20]
    codes = finite_codes(rng, (B, 50, D_QK))
    sc = rng.uniform(1e-3, 2e-2, (B, 50)).astype(np.float32)
    q = om.f64_to_bf16_bits(rng.standard_normal((B, q_len, h, D_QK)))
    ql = np.array([4, 1, 0], dtype=np.int32)
    o, lse = om.mla_decode_fp8(q, codes, sc, lens, scale=SCALE, causal=True, q_lens=ql)
    for b in range(B):
        if ql[b] == 0:
            assert np.all(o[b] == 0) and np.all(lse[b] == -np.inf)
            continue
        ob, lb = om.mla_decode_fp8(q[b:b + 1, :ql[b]], codes[b:b + 1], sc[b:b + 1], lens[b:b + 1], scale=SCALE,
                                   causal=True)
        np.testing.assert_array_equal(o[b, :ql[b]], ob[0])
        np.testing.assert_array_equal(lse[b, :ql[b]], lb[0])
        assert np.all(o[b, ql[b]:] == 0) and np.all(lse[b, ql[b]:] == -np.inf)


def test_generator_quantisation_reconstructs_within_e4m3_rounding():
    from mla_decode_attention_etap_b200 import workloads as W
    w = W.make_workload(2, 16, [300, 77], seed=9, kv_dtype="e4m3")
    kv = w.kv.float().numpy().astype(np.float64)
    rec = torch_e4m3(w.kv8.numpy()) * w.kv_scale.numpy()[..., None].astype(np.float64)
    # E4M3 keeps 4 significant bits: relative error <= 2^-4 above the subnormal range
    amax = np.abs(kv).max(axis=-1, keepdims=True)
    err = np.abs(rec - kv)
    assert np.all(err <= np.maximum(np.abs(kv) * 2.0 ** -4, amax / 448 * 2.0 ** -10) + 1e-30)
    assert np.allclose(np.abs(rec).max(axis=-1), amax[..., 0], rtol=2.0 ** -4)
