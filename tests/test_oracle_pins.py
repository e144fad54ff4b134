"""Pins for the fp64 oracle (CPU only).

The oracle is checked against facts fixed by the mathematics of the definition
(FlashMLA-ETAP technical summary, Methodology: S = Q K^T, P = softmax(S),
O = P V and its transposed ETAP form), not against itself:

* closed forms: one cached row, equal scores, Q = 0, a hand-derived two-row case
  (``tests/golden/closed_form_two_token.json``);
* brute force in exact rational arithmetic plus 40-digit ``decimal`` exp on tiny inputs;
* invariances: KV row permutation, paged == contiguous, causal == non-causal on the
  visible prefix, log-sum-exp merge of disjoint KV ranges, a constant score shift.

Every pin runs against the two C forms and the numpy form.  ``MUTANTS`` are
deliberately wrong variants (a dropped term, a wrong index, a transposed
operand...); each must fail at least one pin, which shows the pins have teeth.
"""

from __future__ import annotations

import json
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

from oracle import mla_oracle as om

D_QK, D_V, PAGE = 576, 512, 64
SCALE = 1.0 / 24.0
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_bits(rng, shape, scale=1.0):
    return om.f64_to_bf16_bits(rng.standard_normal(shape) * scale)


def to_paged(kv_bits, seqlens, rng, page=PAGE):
    """Scatter contiguous rows [B, Lmax, 576] into a shuffled paged pool."""
    B = kv_bits.shape[0]
    nblk = [(int(L) + page - 1) // page for L in seqlens]
    total = sum(nblk)
    perm = rng.permutation(total)
    pool = np.zeros((total, page, D_QK), dtype=np.uint16)
    bt = np.full((B, max(nblk)), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        for i in range(nblk[b]):
            blk = perm[off + i]
            bt[b, i] = blk
            rows = kv_bits[b, i * page:(i + 1) * page]
            pool[blk, :rows.shape[0]] = rows
        off += nblk[b]
    return pool, bt


# ---------------------------------------------------------------------------
# implementations under test
# ---------------------------------------------------------------------------
def impl_c(q, kv, sl, bt=None, scale=SCALE, causal=False):
    return om.mla_decode(q, kv, sl, bt, scale, causal)


def impl_c_etap(q, kv, sl, bt=None, scale=SCALE, causal=False):
    return om.mla_decode_etap(q, kv, sl, bt, scale, causal)


def impl_numpy(q, kv, sl, bt=None, scale=SCALE, causal=False):
    return om.mla_decode_numpy(q, kv, sl, bt, scale, causal)


REAL = {"c": impl_c, "c_etap": impl_c_etap, "numpy": impl_numpy}


def _mutant(kind):
    """numpy oracle with one planted mistake (test-only)."""

    def run(q_bits, kv_bits, sl, bt=None, scale=SCALE, causal=False):
        q = om.bf16_bits_to_f64(q_bits)
        kv = om.bf16_bits_to_f64(kv_bits)
        B, q_len, h, _ = q.shape
        o = np.zeros((B, q_len, h, D_V))
        lse = np.zeros((B, q_len, h))
        for b in range(B):
            L = int(sl[b])
            if bt is not None:
                page = kv.shape[1]
                nb = (L + page - 1) // page
                if kind == "page_index":
                    idx = [int(bt[b, min(i, nb - 1)]) for i in range(nb)]
                    rows = kv[np.asarray(idx)].transpose(1, 0, 2).reshape(nb * page, D_QK)[:L]
                else:
                    rows = kv[np.asarray(bt[b, :nb], dtype=np.int64)].reshape(nb * page, D_QK)[:L]
            else:
                rows = kv[b, :L]
            for t in range(q_len):
                if causal:
                    vis = max(L - q_len + t + (0 if kind == "causal_off_by_one" else 1), 0)
                else:
                    vis = L
                if vis == 0:
                    lse[b, t] = -math.inf
                    continue
                K = rows[:vis]
                qq = q[b, t]
                if kind == "head_order":
                    qq = q[b].transpose(1, 0, 2).reshape(q_len * h, D_QK)[t * h:(t + 1) * h]
                if kind == "drop_rope":
                    S = scale * (qq[:, :D_V] @ K[:, :D_V].T)
                elif kind == "no_scale":
                    S = qq @ K.T
                else:
                    S = scale * (qq @ K.T)
                m = S.max(axis=1, keepdims=True)
                E = np.exp(S - m)
                den = E.sum(axis=1, keepdims=True)
                P = E / den
                if kind == "softmax_over_heads":
                    Eh = np.exp(S - S.max(axis=0, keepdims=True))
                    P = Eh / Eh.sum(axis=0, keepdims=True)
                if kind == "no_normalise":
                    P = E
                V = K[:, D_QK - D_V:] if kind == "v_wrong_columns" else K[:, :D_V]
                o[b, t] = P @ V
                if kind == "lse_log2":
                    lse[b, t] = ((m + np.log2(den)))[:, 0]
                elif kind == "lse_no_max":
                    lse[b, t] = np.log(den)[:, 0]
                else:
                    lse[b, t] = (m + np.log(den))[:, 0]
        return o, lse

    return run


MUTANTS = ["drop_rope", "no_scale", "softmax_over_heads", "no_normalise", "v_wrong_columns",
           "lse_log2", "lse_no_max", "causal_off_by_one", "head_order", "page_index"]


# ---------------------------------------------------------------------------
# exact brute force
# ---------------------------------------------------------------------------
def brute_force(q_bits, kv_bits, sl, scale_frac=Fraction(1, 24), causal=False, digits=40):
    """Exact scores (bf16 values are dyadic rationals), 40-digit exp, no fp64 anywhere."""
    getcontext().prec = digits
    q = [[[[Fraction(float(x)) for x in row] for row in hh] for hh in tt] for tt in om.bf16_bits_to_f64(q_bits)]
    kv = om.bf16_bits_to_f64(kv_bits)
    B, q_len, h = len(q), len(q[0]), len(q[0][0])
    o = np.zeros((B, q_len, h, D_V))
    lse = np.zeros((B, q_len, h))
    for b in range(B):
        L = int(sl[b])
        K = [[Fraction(float(x)) for x in kv[b, j]] for j in range(L)]
        for t in range(q_len):
            vis = max(L - q_len + t + 1, 0) if causal else L
            for hd in range(h):
                if vis == 0:
                    lse[b, t, hd] = -math.inf
                    continue
                s = [scale_frac * sum(a * c for a, c in zip(q[b][t][hd], K[j])) for j in range(vis)]
                m = max(s)
                e = [(Decimal(x.numerator) / Decimal(x.denominator) - Decimal(m.numerator) / Decimal(m.denominator)).exp()
                     for x in s]
                den = sum(e)
                for d in range(D_V):
                    o[b, t, hd, d] = float(sum(e[j] * Decimal(K[j][d].numerator) / Decimal(K[j][d].denominator)
                                               for j in range(vis)) / den)
                lse[b, t, hd] = float(Decimal(m.numerator) / Decimal(m.denominator) + den.ln())
    return o, lse


# ---------------------------------------------------------------------------
# pins: each takes an implementation and raises AssertionError on violation
# ---------------------------------------------------------------------------
def pin_single_row(impl):
    rng = np.random.default_rng(11)
    q = rand_bits(rng, (2, 1, 3, D_QK))
    kv = rand_bits(rng, (2, 1, D_QK))
    sl = np.array([1, 1], np.int32)
    o, lse = impl(q, kv, sl)
    qf, kf = om.bf16_bits_to_f64(q), om.bf16_bits_to_f64(kv)
    for b in range(2):
        for hd in range(3):
            np.testing.assert_array_equal(o[b, 0, hd], kf[b, 0, :D_V])
            exact = Fraction(sum(Fraction(float(a)) * Fraction(float(c)) for a, c in zip(qf[b, 0, hd], kf[b, 0])), 24)
            assert abs(lse[b, 0, hd] - float(exact)) <= 1e-12 * max(1.0, abs(float(exact)))


def pin_equal_scores(impl):
    rng = np.random.default_rng(12)
    B, h, L = 1, 4, 37
    qf = rng.standard_normal((B, 1, h, D_QK))
    qf[..., :D_V] = 0.0                       # only the last 64 query columns are non-zero
    kvf = rng.standard_normal((B, L, D_QK))
    kvf[:, :, D_V:] = rng.standard_normal(D_QK - D_V)  # every row shares its last 64 columns
    q, kv = om.f64_to_bf16_bits(qf), om.f64_to_bf16_bits(kvf)
    o, lse = impl(q, kv, np.array([L], np.int32))
    qd, kd = om.bf16_bits_to_f64(q), om.bf16_bits_to_f64(kv)
    mean_v = kd[0, :, :D_V].mean(axis=0)
    for hd in range(h):
        s = SCALE * float(qd[0, 0, hd] @ kd[0, 0])
        np.testing.assert_allclose(o[0, 0, hd], mean_v, rtol=0, atol=1e-12)
        assert abs(lse[0, 0, hd] - (s + math.log(L))) < 1e-12


def pin_zero_query(impl):
    rng = np.random.default_rng(13)
    L = 50
    q = np.zeros((1, 1, 2, D_QK), np.uint16)
    kv = rand_bits(rng, (1, L, D_QK))
    o, lse = impl(q, kv, np.array([L], np.int32))
    mean_v = om.bf16_bits_to_f64(kv)[0, :, :D_V].mean(axis=0)
    np.testing.assert_allclose(o[0, 0, 0], mean_v, atol=1e-12, rtol=0)
    assert abs(lse[0, 0, 1] - math.log(L)) < 1e-12


def pin_closed_form_golden(impl):
    with open(os.path.join(GOLDEN, "closed_form_two_token.json")) as f:
        g = json.load(f)
    q = np.zeros((1, 1, 1, D_QK))
    for c, v in g["q_nonzero"]:
        q[0, 0, 0, c] = v
    kv = np.zeros((1, 2, D_QK))
    for j, row in enumerate(g["kv_rows_nonzero"]):
        for c, v in row:
            kv[0, j, c] = v
    o, lse = impl(om.f64_to_bf16_bits(q), om.f64_to_bf16_bits(kv), np.array([2], np.int32), scale=1.0 / 24.0)
    env = {"e": math.e, "log": math.log}
    expect = np.zeros(D_V)
    for c, expr in g["expected_o_nonzero"]:
        expect[c] = eval(expr, {}, env)
    np.testing.assert_allclose(o[0, 0, 0], expect, rtol=1e-14, atol=1e-15)
    assert abs(lse[0, 0, 0] - eval(g["expected_lse"], {}, env)) < 1e-14


def pin_brute_force(impl):
    rng = np.random.default_rng(14)
    q = rand_bits(rng, (2, 2, 2, D_QK))
    kv = rand_bits(rng, (2, 5, D_QK), scale=1.5)
    sl = np.array([5, 3], np.int32)
    for causal in (False, True):
        o, lse = impl(q, kv, sl, causal=causal)
        ob, lb = brute_force(q, kv, sl, causal=causal)
        np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)


def pin_causal_prefix(impl):
    rng = np.random.default_rng(15)
    q_len, h, L = 3, 2, 40
    q = rand_bits(rng, (1, q_len, h, D_QK))
    kv = rand_bits(rng, (1, L, D_QK))
    o, lse = impl(q, kv, np.array([L], np.int32), causal=True)
    for t in range(q_len):
        vis = L - q_len + t + 1
        o1, l1 = impl(q[:, t:t + 1].copy(), kv[:, :vis].copy(), np.array([vis], np.int32))
        np.testing.assert_allclose(o[:, t], o1[:, 0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, t], l1[:, 0], rtol=0, atol=1e-13)


def pin_paged_equals_contiguous(impl):
    rng = np.random.default_rng(16)
    sl = np.array([130, 64, 5], np.int32)
    q = rand_bits(rng, (3, 1, 2, D_QK))
    kv = rand_bits(rng, (3, 130, D_QK))
    pool, bt = to_paged(kv, sl, rng)
    o1, l1 = impl(q, kv, sl)
    o2, l2 = impl(q, pool, sl, bt)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def pin_permutation(impl):
    rng = np.random.default_rng(17)
    L = 33
    q = rand_bits(rng, (1, 2, 2, D_QK))
    kv = rand_bits(rng, (1, L, D_QK))
    o1, l1 = impl(q, kv, np.array([L], np.int32))
    o2, l2 = impl(q, kv[:, rng.permutation(L)].copy(), np.array([L], np.int32))
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def pin_split_merge(impl):
    rng = np.random.default_rng(18)
    L, a = 77, 30
    q = rand_bits(rng, (1, 1, 3, D_QK))
    kv = rand_bits(rng, (1, L, D_QK))
    o, lse = impl(q, kv, np.array([L], np.int32))
    oa, la = impl(q, kv[:, :a].copy(), np.array([a], np.int32))
    ob, lb = impl(q, kv[:, a:].copy(), np.array([L - a], np.int32))
    for hd in range(3):
        om_, lm = om.lse_merge(np.stack([oa[0, 0, hd], ob[0, 0, hd]]), np.array([la[0, 0, hd], lb[0, 0, hd]]))
        np.testing.assert_allclose(om_, o[0, 0, hd], rtol=0, atol=1e-13)
        assert abs(lm - lse[0, 0, hd]) < 1e-13


def pin_score_shift(impl):
    rng = np.random.default_rng(19)
    L = 21
    qf = rng.standard_normal((1, 1, 1, D_QK))
    kvf = rng.standard_normal((1, L, D_QK))
    u = np.zeros(D_QK - D_V)
    u[0] = 1.0
    kvf[:, :, D_V:] = u                      # every row: last 64 columns = e_0
    q1, kv = om.f64_to_bf16_bits(qf), om.f64_to_bf16_bits(kvf)
    qf2 = om.bf16_bits_to_f64(q1).copy()
    qf2[..., D_V] += 3.0                     # shifts every score by 3/24 exactly
    q2 = om.f64_to_bf16_bits(qf2)
    delta = (om.bf16_bits_to_f64(q2) - om.bf16_bits_to_f64(q1))[0, 0, 0, D_V] / 24.0
    o1, l1 = impl(q1, kv, np.array([L], np.int32))
    o2, l2 = impl(q2, kv, np.array([L], np.int32))
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-13)
    assert abs(l2[0, 0, 0] - l1[0, 0, 0] - delta) < 1e-13


PINS = [pin_single_row, pin_equal_scores, pin_zero_query, pin_closed_form_golden, pin_brute_force,
        pin_causal_prefix, pin_paged_equals_contiguous, pin_permutation, pin_split_merge, pin_score_shift]


@pytest.mark.parametrize("name", sorted(REAL))
@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin_holds(pin, name):
    pin(REAL[name])


@pytest.mark.parametrize("kind", MUTANTS)
def test_mutant_fails_a_pin(kind):
    impl = _mutant(kind)
    failed = []
    for pin in PINS:
        try:
            pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {kind!r} passed every pin"


def test_unmutated_reference_passes_all_pins():
    impl = _mutant("none")
    for pin in PINS:
        pin(impl)


def test_forms_agree_on_random_inputs():
    """Standard form, transposed ETAP form and numpy form agree on mixed shapes."""
    rng = np.random.default_rng(20)
    sl = np.array([200, 1, 129, 64], np.int32)
    q = rand_bits(rng, (4, 4, 3, D_QK))
    kv = rand_bits(rng, (4, 200, D_QK))
    for causal in (False, True):
        ref = impl_c(q, kv, sl, causal=causal)
        for other in (impl_c_etap, impl_numpy):
            o, lse = other(q, kv, sl, causal=causal)
            np.testing.assert_allclose(o, ref[0], rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse, ref[1], rtol=0, atol=1e-13)


def test_empty_sequence_and_fully_masked_columns():
    rng = np.random.default_rng(21)
    q = rand_bits(rng, (2, 4, 2, D_QK))
    kv = rand_bits(rng, (2, 8, D_QK))
    sl = np.array([0, 2], np.int32)
    for impl in REAL.values():
        o, lse = impl(q, kv, sl, causal=True)
        assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
        # L=2, q_len=4: tokens 0 and 1 see no row, tokens 2 and 3 see 1 and 2 rows
        assert np.all(np.isneginf(lse[1, :2])) and np.all(o[1, :2] == 0)
        np.testing.assert_array_equal(o[1, 2, 0], om.bf16_bits_to_f64(kv)[1, 0, :D_V])


def test_lse_merge_all_empty():
    o, lse = om.lse_merge(np.zeros((3, D_V)), np.array([-math.inf] * 3))
    assert lse == -math.inf and np.all(o == 0)


# ---------------------------------------------------------------- ragged multi-token decode
# q_lens[b] real query tokens in sequence b; the q_lens[b] new tokens are the last q_lens[b] cache
# rows.  Pinned against the uniform form (itself pinned above): sequence b of a ragged batch is
# the uniform decode of that sequence alone with q_len = q_lens[b], and padding tokens see nothing.

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("ragged", ["c", "numpy"])
def test_ragged_equals_each_sequence_decoded_alone(causal, ragged):
    rng = np.random.default_rng(30)
    sl = np.array([300, 5, 129, 2], np.int32)
    q_lens = np.array([1, 4, 2, 3], np.int32)
    q = rand_bits(rng, (4, 4, 3, D_QK))
    kv = rand_bits(rng, (4, 300, D_QK))
    fn = om.mla_decode if ragged == "c" else om.mla_decode_numpy
    o, lse = fn(q, kv, sl, None, SCALE, causal, q_lens=q_lens)
    for b in range(4):
        qb = int(q_lens[b])
        o1, l1 = om.mla_decode(q[b:b + 1, :qb], kv[b:b + 1], sl[b:b + 1], None, SCALE, causal)
        np.testing.assert_allclose(o[b, :qb], o1[0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[b, :qb], l1[0], rtol=0, atol=1e-13)
        assert np.all(o[b, qb:] == 0) and np.all(np.isneginf(lse[b, qb:]))


def test_ragged_with_full_lengths_is_the_uniform_decode():
    rng = np.random.default_rng(31)
    sl = np.array([70, 130], np.int32)
    q = rand_bits(rng, (2, 3, 2, D_QK))
    kv = rand_bits(rng, (2, 130, D_QK))
    for causal in (False, True):
        ref = om.mla_decode(q, kv, sl, None, SCALE, causal)
        got = om.mla_decode(q, kv, sl, None, SCALE, causal, q_lens=np.array([3, 3], np.int32))
        np.testing.assert_array_equal(got[0], ref[0])
        np.testing.assert_array_equal(got[1], ref[1])


def test_ragged_causal_offset_uses_the_sequence_own_token_count():
    """Token 0 of a sequence with 2 new tokens sees L-1 rows (not L-q_max+1): with q_max = 4 and
    L = 6 a wrong offset would give it 3 rows; check the visible count through a one-hot V."""
    L, h = 6, 1
    q = np.zeros((1, 4, h, D_QK), np.uint16)                   # Q = 0: equal scores, O = mean of visible V
    kv = np.zeros((1, L, D_QK), np.float64)
    kv[0, :, 0] = 1.0                                          # every visible row contributes 1 to O[0]
    kv[0, :, 1] = np.arange(L)                                 # O[1] = mean row index of the visible rows
    kvb = om.f64_to_bf16_bits(kv)
    o, lse = om.mla_decode(q, kvb, np.array([L], np.int32), None, SCALE, True, q_lens=np.array([2], np.int32))
    # token 0 sees rows 0..4 (mean 2.0, LSE ln 5), token 1 sees rows 0..5 (mean 2.5, LSE ln 6)
    np.testing.assert_allclose(o[0, 0, 0, 1], 2.0, atol=1e-12)
    np.testing.assert_allclose(o[0, 1, 0, 1], 2.5, atol=1e-12)
    np.testing.assert_allclose(lse[0, :2, 0], [math.log(5), math.log(6)], atol=1e-12)
    assert np.all(np.isneginf(lse[0, 2:]))
