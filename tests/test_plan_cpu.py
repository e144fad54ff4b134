"""The split-KV schedules (host mirror of the device plan kernel; both come from
the same shared source): coverage, balance, split bookkeeping, and the choice of
column-group width for the bf16 cache's M = 256 kernel."""

from __future__ import annotations

import numpy as np
import pytest

import mla_decode_attention_etap_b200 as m

SINGLE_P_MIN_ROWS = 8192  # plan_core.h: one bf16 P term only when every nonempty sequence is this long


def units(L, rows):
    return 0 if L <= 0 else (L + rows - 1) // rows


def end_cost(rows):
    """Units a sequence end counts for when the ranges are cut (plan_core.h: end_cost_units)."""
    return 4 if rows == 128 else 2


def cost_cut(lens, rows, ctas):
    """The cost-balanced cut written out directly: the cost axis holds each nonempty sequence's units
    followed by end_cost(rows) end positions; it is cut into min(T, ctas) near-equal pieces, and each
    cut lands on the unit it falls on (or, among a sequence's end positions, on its last boundary)."""
    us = [units(int(L), rows) for L in lens]
    T = sum(us)
    used = min(T, ctas)
    C = sum(u + (end_cost(rows) if u else 0) for u in us)
    begins = []
    for c in range(ctas):
        if c >= used:
            begins.append(T)
            continue
        x = C * c // used
        g = f = 0
        for u in us:
            gend = g + u + (end_cost(rows) if u else 0)
            if u and g <= x < gend:
                begins.append(f + min(x - g, u))
                break
            g, f = gend, f + u
    return [(begins[c], begins[c + 1] if c + 1 < ctas else T) for c in range(ctas)]


def expected_grouping(lens, q, h, n_sms, schedule):
    """(unit_rows, group_cols, groups, ctas) as the pages' decode path is laid out here."""
    ncols = q * h
    if schedule == 0 or ncols <= 16:
        gc = 16 if ncols <= 16 else 32
        rows = 128
    else:
        nonempty = [int(L) for L in lens if L > 0]
        single = ncols > 64 and bool(nonempty) and min(nonempty) >= SINGLE_P_MIN_ROWS
        gc = 128 if single else 64
        rows = 256
    groups = (ncols + gc - 1) // gc
    return rows, gc, groups, max(1, n_sms // 2 // groups)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("schedule", [0, 1])
@pytest.mark.parametrize("n_sms,h,q", [(148, 16, 1), (148, 128, 1), (148, 16, 4), (7, 16, 1), (1, 16, 1), (300, 16, 1),
                                       (148, 32, 1), (148, 16, 16)])
def test_schedule_invariants(seed, schedule, n_sms, h, q):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 70))
    lens = rng.integers(0, 70000, B)
    lens[rng.random(B) < 0.2] = 0
    if seed % 2:  # half the batches long enough for single-term P groups
        lens = np.where(lens > 0, lens + SINGLE_P_MIN_ROWS, 0)
    ranges, info, ctas, groups, rows, gcols = m.mla_decode_plan_host(lens, q, h, n_sms, schedule)
    assert (rows, gcols, groups, ctas) == expected_grouping(lens, q, h, n_sms, schedule)
    T = sum(units(int(L), rows) for L in lens)
    # the unit ranges tile [0, T) in order, cut by cost (each sequence end counts as extra units)
    assert ranges[0, 0] == 0 and ranges[-1, 1] == T
    assert np.all(ranges[1:, 0] == ranges[:-1, 1])
    assert [tuple(r) for r in ranges.tolist()] == cost_cut(lens, rows, ctas)
    sizes = ranges[:, 1] - ranges[:, 0]
    used = min(ctas, T)
    assert np.all(sizes[used:] == 0)
    if used:
        # a range's units plus the end costs it carries stay within one end cost + 1 of the fair share
        ends = np.zeros(ctas, np.int64)
        off = 0
        for L in lens:
            u = units(int(L), rows)
            if u:
                last = off + u - 1
                ends[int(np.searchsorted(ranges[:, 1], last, side="right"))] += 1
            off += u
        cost = sizes + end_cost(rows) * ends
        C = T + end_cost(rows) * int(sum(1 for L in lens if units(int(L), rows)))
        assert np.all(np.abs(cost[:used] - C / used) <= end_cost(rows) + 1)
    # per sequence: the units that own some of its rows are exactly [first, first + nsplit)
    off = 0
    slots = 0
    for b, L in enumerate(lens):
        nt = units(int(L), rows)
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
    assert slots <= B + ctas  # the workspace reserves batch + units partial slots


@pytest.mark.parametrize("lens,n_sms", [([129], 148), ([1024], 148), ([3000, 257, 1536], 148), ([5], 16),
                                         ([0, 0, 1], 148), ([300, 1100, 129], 18)])
@pytest.mark.parametrize("h", [16, 64])
def test_fewer_units_than_ctas(lens, n_sms, h):
    """Regression: idle units must not sit between the splits of one sequence."""
    ranges, info, ctas, _, rows, _ = m.mla_decode_plan_host(lens, 1, h, n_sms)
    sizes = ranges[:, 1] - ranges[:, 0]
    for b, L in enumerate(lens):
        if units(L, rows) == 0:
            continue
        first, ns = info[b, 1], info[b, 2]
        assert np.all(sizes[first:first + ns] > 0)
        assert ns == min(units(L, rows), ns)


def test_headline_shape_balance():
    """16 x 512 tiles over 74 CTA pairs: a pair that holds a sequence end takes about 4 tiles fewer."""
    ranges, info, ctas, groups, rows, gcols = m.mla_decode_plan_host([65536] * 16, 1, 16, 148)
    assert (ctas, groups, rows, gcols) == (74, 1, 128, 16)
    sizes = ranges[:, 1] - ranges[:, 0]
    assert sizes.sum() == 8192 and sizes.min() >= 107 and sizes.max() <= 112
    ends = [int(np.searchsorted(ranges[:, 1], 512 * (b + 1) - 1, side="right")) for b in range(16)]
    others = np.setdiff1d(np.arange(74), ends)
    assert sizes[ends].mean() + 3 < sizes[others].mean()
    assert np.all(info[:, 2] >= 4)


def test_h128_groups_depend_on_the_shortest_sequence():
    """128 heads: one 128-column group per unit (74 units) when every sequence holds >= 8192 rows,
    else two 64-column groups (37 units each); empty sequences do not count."""
    long = [8192, 20000, 0, 32768]
    assert m.mla_decode_plan_host(long, 1, 128, 148)[2:] == (74, 1, 256, 128)
    short = [8191, 20000, 32768]
    assert m.mla_decode_plan_host(short, 1, 128, 148)[2:] == (37, 2, 256, 64)
    # the FP8 cache keeps 32-column groups of 128-row tiles
    assert m.mla_decode_plan_host(long, 1, 128, 148, schedule=0)[2:] == (18, 4, 128, 32)
    # q_len = 4 at 16 heads: one 64-column group, whatever the lengths
    assert m.mla_decode_plan_host([32768] * 16, 4, 16, 148)[2:] == (74, 1, 256, 64)


def test_workspace_covers_both_groupings():
    """The workspace is sized before the plan picks the grouping: it holds the partial slots and merge
    counters of the larger of the two."""
    for B, q, h in ((32, 1, 128), (16, 4, 16), (3, 16, 16), (64, 1, 16)):
        need = m.mla_decode_workspace_size(B, q, h, 148)
        ncols = q * h
        slots_max = B + max(expected_grouping([1], q, h, 148, 1)[3], expected_grouping([10 ** 6], q, h, 148, 1)[3],
                            expected_grouping([1], q, h, 148, 0)[3])
        assert need >= 4 * slots_max * ncols * 512
