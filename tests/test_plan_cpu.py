"""The split-KV schedule (host mirror of the device plan kernel; both come from
the same shared source): coverage, balance and split bookkeeping."""

from __future__ import annotations

import numpy as np
import pytest

import mla_decode_attention_etap_b200 as m


def tiles(L):
    return 0 if L <= 0 else (L + 127) // 128


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("n_sms,h,q", [(148, 16, 1), (148, 128, 1), (148, 16, 4), (7, 16, 1), (1, 16, 1), (300, 16, 1)])
def test_schedule_invariants(seed, n_sms, h, q):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 70))
    lens = rng.integers(0, 70000, B)
    lens[rng.random(B) < 0.2] = 0
    ranges, info, ctas, groups = m.mla_decode_plan_host(lens, q, h, n_sms)
    ncols = q * h
    assert groups == (1 if ncols <= 16 else (ncols + 31) // 32)
    assert ctas == max(1, n_sms // 2 // groups)  # one work unit per SM pair
    T = sum(tiles(int(L)) for L in lens)
    # the CTA ranges tile [0, T) in order; the working CTAs come first, each with
    # at least one tile, sizes within 1 of each other; idle CTAs (only when T < ctas) come last
    assert ranges[0, 0] == 0 and ranges[-1, 1] == T
    assert np.all(ranges[1:, 0] == ranges[:-1, 1])
    sizes = ranges[:, 1] - ranges[:, 0]
    used = min(ctas, T)
    assert np.all(sizes[:used] >= 1) and np.all(sizes[used:] == 0)
    if used:
        assert sizes[:used].max() - sizes[:used].min() <= 1
    # per sequence: the CTAs that own some of its tiles are exactly [first, first + nsplit)
    off = 0
    slots = 0
    for b, L in enumerate(lens):
        nt = tiles(int(L))
        assert info[b, 0] == nt
        if nt == 0:
            assert info[b, 2] == 0
        else:
            over = [c for c in range(ctas) if sizes[c] > 0 and ranges[c, 0] < off + nt and ranges[c, 1] > off]
            assert info[b, 1] == over[0] and info[b, 2] == len(over)
            assert over == list(range(over[0], over[0] + len(over)))
        assert info[b, 3] == slots
        if info[b, 2] >= 2:
            slots += info[b, 2]
        off += nt
    assert slots <= B + ctas  # the workspace reserves batch + ctas partial slots


@pytest.mark.parametrize("lens,n_sms", [([129], 148), ([1024], 148), ([3000, 257, 1536], 148), ([5], 16),
                                         ([0, 0, 1], 148), ([300, 1100, 129], 18)])
def test_fewer_tiles_than_ctas(lens, n_sms):
    """Regression: idle CTAs must not sit between the splits of one sequence."""
    ranges, info, ctas, _ = m.mla_decode_plan_host(lens, 1, 16, n_sms)
    sizes = ranges[:, 1] - ranges[:, 0]
    for b, L in enumerate(lens):
        if tiles(L) == 0:
            continue
        first, ns = info[b, 1], info[b, 2]
        assert np.all(sizes[first:first + ns] > 0)
        assert ns == min(tiles(L), ns)


def test_headline_shape_balance():
    ranges, info, ctas, groups = m.mla_decode_plan_host([65536] * 16, 1, 16, 148)
    assert ctas == 74 and groups == 1
    sizes = ranges[:, 1] - ranges[:, 0]
    assert sizes.min() == 110 and sizes.max() == 111
    assert np.all(info[:, 2] >= 5)
