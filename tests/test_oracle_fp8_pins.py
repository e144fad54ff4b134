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


# ---------------------------------------------------------------------------
# The same pins as functions of an implementation, run on both oracle forms and on deliberately
# wrong variants (a mistake planted in a test-only numpy decode): every variant must fail a pin.
def _widen(codes, kind=""):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e, m = (c >> 3) & 15, c & 7
    bias = 8.0 if kind == "e4m3_bias" else 7.0
    if kind == "e4m3_subnormal_as_normal":
        mag = (1.0 + m / 8.0) * np.exp2(np.maximum(e, 1) - bias)
    else:
        mag = np.where(e == 0, m / 8.0 * 2.0 ** (1 - bias), (1.0 + m / 8.0) * np.exp2(e - bias))
    return mag if kind == "sign_dropped" else np.where(c & 0x80, -mag, mag)


def _mutant8(kind):
    def run(q_bits, codes, sc, sl, block_table=None, scale=SCALE, causal=False, q_lens=None):
        q = om.bf16_bits_to_f64(q_bits)
        w = _widen(codes, kind)
        s = np.asarray(sc, dtype=np.float64)
        k_scale = np.ones_like(s) if kind == "no_row_scale" else (s * s if kind == "scale_squared" else s)
        v_scale = np.ones_like(s) if kind in ("no_row_scale", "scale_on_scores_only") else k_scale
        B, q_len, h, _ = q.shape
        o = np.zeros((B, q_len, h, D_V))
        lse = np.zeros((B, q_len, h))
        for b in range(B):
            L = int(sl[b])
            if block_table is not None:
                nb = (L + PAGE - 1) // PAGE
                idx = np.asarray(block_table[b, :nb], dtype=np.int64)
                # the planted paging mistake reads the scales of the logical, not the physical, block
                sidx = np.arange(nb) if kind == "paged_scale_logical" else idx
                rows = w[idx].reshape(nb * PAGE, D_QK)[:L]
                krows = rows * k_scale[sidx].reshape(-1)[:L, None]
                vrows = rows * v_scale[sidx].reshape(-1)[:L, None]
            else:
                krows, vrows = w[b, :L] * k_scale[b, :L, None], w[b, :L] * v_scale[b, :L, None]
            for t in range(q_len):
                vis = max(L - q_len + t + 1, 0) if causal else L
                if vis == 0:
                    lse[b, t] = -math.inf
                    continue
                S = scale * (q[b, t] @ krows[:vis].T)
                mx = S.max(axis=1, keepdims=True)
                E = np.exp(S - mx)
                den = E.sum(axis=1, keepdims=True)
                o[b, t] = (E / den) @ vrows[:vis, :D_V]
                lse[b, t] = (mx + np.log(den))[:, 0]
        return o, lse
    return run


def _pin_codes_table(impl):
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    kv = np.zeros((1, 1, D_QK), dtype=np.uint8)
    kv[0, 0, :254] = codes
    q = om.f64_to_bf16_bits(np.random.default_rng(20).standard_normal((1, 1, 2, D_QK)))
    o, _ = impl(q, kv, np.ones((1, 1), np.float32), [1], scale=SCALE)
    np.testing.assert_array_equal(o[0, 0, 0, :254], torch_e4m3(codes))


def _pin_pow2_bf16(impl):
    rng = np.random.default_rng(21)
    codes = finite_codes(rng, (2, 70, D_QK))
    sc = np.exp2(rng.integers(-12, -3, (2, 70))).astype(np.float32)
    bits = om.f64_to_bf16_bits(torch_e4m3(codes) * sc[..., None].astype(np.float64))
    q = om.f64_to_bf16_bits(rng.standard_normal((2, 1, 4, D_QK)))
    o8, l8 = impl(q, codes, sc, [70, 33], scale=SCALE)
    ob, lb = om.mla_decode(q, bits, [70, 33], scale=SCALE)
    np.testing.assert_allclose(o8, ob, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l8, lb, rtol=0, atol=1e-12)


def _pin_zero_query(impl):
    rng = np.random.default_rng(22)
    codes = finite_codes(rng, (1, 37, D_QK))
    sc = rng.uniform(1e-3, 1e-2, (1, 37)).astype(np.float32)
    o, lse = impl(np.zeros((1, 1, 2, D_QK), np.uint16), codes, sc, [37], scale=SCALE)
    v = torch_e4m3(codes[0, :, :D_V]) * sc[0][:, None].astype(np.float64)
    np.testing.assert_allclose(o[0, 0, 0], v.mean(axis=0), rtol=1e-12, atol=1e-16)
    np.testing.assert_allclose(lse[0, 0], math.log(37), rtol=1e-14)


def _pin_paged(impl):
    rng = np.random.default_rng(23)
    lens = [130, 64]
    codes = finite_codes(rng, (2, 130, D_QK))
    sc = rng.uniform(1e-3, 2e-2, (2, 130)).astype(np.float32)
    q = om.f64_to_bf16_bits(rng.standard_normal((2, 1, 4, D_QK)))
    nblk = [3, 1]
    perm = rng.permutation(4)
    pool = np.zeros((4, PAGE, D_QK), np.uint8)
    pool_sc = np.ones((4, PAGE), np.float32)
    bt = np.full((2, 3), -1, np.int32)
    off = 0
    for b in range(2):
        for i in range(nblk[b]):
            blk = perm[off + i]
            bt[b, i] = blk
            n = min(PAGE, 130 - i * PAGE)
            pool[blk, :n] = codes[b, i * PAGE:i * PAGE + n]
            pool_sc[blk, :n] = sc[b, i * PAGE:i * PAGE + n]
        off += nblk[b]
    oc, lc = impl(q, codes, sc, lens, scale=SCALE)
    op, lp = impl(q, pool, pool_sc, lens, block_table=bt, scale=SCALE)
    np.testing.assert_allclose(op, oc, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lp, lc, rtol=0, atol=1e-12)


PINS8 = {"codes_table": _pin_codes_table, "pow2_equals_bf16": _pin_pow2_bf16, "zero_query": _pin_zero_query,
         "paged": _pin_paged}
IMPLS8 = {"c": om.mla_decode_fp8, "numpy": om.mla_decode_fp8_numpy, "test_decode": _mutant8("")}
MUTANTS8 = ["e4m3_bias", "e4m3_subnormal_as_normal", "sign_dropped", "no_row_scale", "scale_squared",
            "scale_on_scores_only", "paged_scale_logical"]


@pytest.mark.parametrize("pin", sorted(PINS8))
@pytest.mark.parametrize("impl", sorted(IMPLS8))
def test_fp8_pin_holds(pin, impl):
    PINS8[pin](IMPLS8[impl])


@pytest.mark.parametrize("kind", MUTANTS8)
def test_fp8_mutant_fails_a_pin(kind):
    failed = []
    for name, pin in PINS8.items():
        try:
            pin(_mutant8(kind))
        except AssertionError:
            failed.append(name)
    assert failed, f"planted mistake {kind!r} passed every pin"
