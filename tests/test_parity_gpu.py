"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, element by element.

Small cases span several 128-row tiles and ragged tails and are compared in
full; the full-size workloads run in the launch configuration of bench.py
(148 SMs) and are compared on sampled sequences the oracle computes one by one.
Tolerance (applied to each compared tensor): RMSE(O) <= 2e-3 RMS(O_ref),
max|dO| <= 1e-2 max|O_ref|, max|dLSE| <= 1e-3.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from mla_decode_attention_etap_b200 import workloads as W
from tests.parity import assert_parity, run_cuda, run_oracle

pytestmark = pytest.mark.gpu


def _poison_padding(w: W.Workload):
    """NaN in every cache row the sequences do not own: the kernel must never let it into O."""
    nan = torch.tensor(float("nan"), dtype=torch.bfloat16)
    if w.block_table is None:
        for b in range(w.batch):
            w.kv[b, int(w.seqlens[b]):] = nan
    else:
        used = set()
        for b in range(w.batch):
            L = int(w.seqlens[b])
            nb = (L + 63) // 64
            for i in range(nb):
                blk = int(w.block_table[b, i])
                used.add(blk)
                if i == nb - 1 and L % 64:
                    w.kv[blk, L % 64:] = nan
        for blk in range(w.kv.shape[0]):
            if blk not in used:
                w.kv[blk] = nan
    return w


def test_b1_h16_l1024():
    w = W.workload_b1_h16_l1024(seed=0)
    o, lse, st, _ = run_cuda(w)
    assert st == 0
    assert_parity(o, lse, *run_oracle(w), what="B=1 h=16 L=1024")


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 127, 128, 129, 511, 512, 513, 1000])
def test_edge_lengths_single_sequence(L):
    w = _poison_padding(W.make_workload(1, 16, [L], seed=L, l_max=L + 200))
    o, lse, st, _ = run_cuda(w)
    assert st == 0
    assert_parity(o, lse, *run_oracle(w), what=f"L={L}")


def test_mixed_lengths_with_empty_sequence_and_nan_padding():
    lens = [0, 1, 129, 700, 64, 2000, 3, 0]
    w = _poison_padding(W.make_workload(len(lens), 16, lens, seed=3))
    o, lse, st, _ = run_cuda(w)
    assert st == 0
    o_ref, lse_ref = run_oracle(w)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    assert_parity(o, lse, o_ref, lse_ref, what="mixed")


@pytest.mark.parametrize("n_sms", [1, 3, 16, 148, 300, 1024])
def test_split_counts(n_sms):
    """From one CTA walking every sequence to many CTAs per sequence (split + combine)."""
    w = W.make_workload(3, 16, [3000, 257, 1536], seed=4)
    o, lse, st, dec = run_cuda(w, n_sms=n_sms)
    assert st == 0
    assert_parity(o, lse, *run_oracle(w), what=f"n_sms={n_sms}")


def test_paged_random_permutation_nan_elsewhere():
    lens = [1, 64, 65, 300, 1234, 4096, 77]
    w = _poison_padding(W.make_workload(len(lens), 16, lens, paged=True, seed=5, extra_blocks=7))
    o, lse, st, _ = run_cuda(w)
    assert st == 0
    assert_parity(o, lse, *run_oracle(w), what="paged")


@pytest.mark.parametrize("L", [2, 5, 100, 131, 700])
def test_causal_q4(L):
    w = W.make_workload(2, 16, [L, L + 37], q_len=4, causal=True, seed=6, spike_frac=0.05)
    o, lse, st, _ = run_cuda(w)
    assert st == 0
    assert_parity(o, lse, *run_oracle(w), what=f"causal L={L}")


def test_causal_shorter_than_q_len():
    w = W.make_workload(1, 16, [2], q_len=4, causal=True, seed=7)
    o, lse, st, _ = run_cuda(w)
    o_ref, lse_ref = run_oracle(w)
    assert np.all(np.isneginf(lse[0, :2])) and np.all(o[0, :2] == 0)
    assert_parity(o, lse, o_ref, lse_ref, what="causal L<q")


def test_h128_paged():
    w = W.make_workload(3, 128, [300, 1100, 129], paged=True, seed=8)
    o, lse, st, _ = run_cuda(w)
    assert st == 0
    assert_parity(o, lse, *run_oracle(w), what="h=128")


def test_odd_column_count():
    """q_len*h not a multiple of 16: the last column group is partly empty."""
    w = W.make_workload(2, 8, [500, 90], q_len=1, seed=9)
    o, lse, st, _ = run_cuda(w)
    assert_parity(o, lse, *run_oracle(w), what="h=8")
    w = W.make_workload(2, 20, [333, 1], q_len=1, seed=10)
    o, lse, st, _ = run_cuda(w)
    assert_parity(o, lse, *run_oracle(w), what="h=20")


def test_spiky_scores_force_rescale():
    """Rows scaled x8 and x64 make running maxima jump (TMEM rescale path)."""
    w = W.make_workload(2, 16, [5000, 3000], seed=11, spike_frac=0.05, spike_scale=8.0)
    o, lse, st, _ = run_cuda(w)
    assert_parity(o, lse, *run_oracle(w), what="spikes x8")
    w = W.make_workload(1, 16, [4000], seed=12)
    w.kv[0, 3500] = (w.kv[0, 3500].float() * 64).to(torch.bfloat16)
    w.kv[0, 100] = (w.kv[0, 100].float() * 16).to(torch.bfloat16)
    o, lse, st, _ = run_cuda(w)
    assert_parity(o, lse, *run_oracle(w), what="spikes x64")


def test_repeat_is_deterministic_and_skip_combine_path():
    w = W.make_workload(2, 16, [4000, 900], seed=13)
    o1, l1, _, dec = run_cuda(w)
    o2, l2, _, _ = run_cuda(w, decoder=dec)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    # fwd without combine, then the separate combine call
    from mla_decode_attention_etap_b200 import FLAG_SKIP_COMBINE, mla_combine
    o3, l3, _, dec3 = run_cuda(w, flags=FLAG_SKIP_COMBINE, poison=False)
    dev = torch.device("cuda")
    o_t = torch.tensor(o3, dtype=torch.bfloat16, device=dev)
    l_t = torch.tensor(l3, dtype=torch.float32, device=dev)
    mla_combine(dec3.workspace, w.batch, w.q_len, w.num_heads, dec3.n_sms, o_t, l_t)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(o_t.float().cpu().numpy(), o1)
    np.testing.assert_array_equal(l_t.cpu().numpy(), l1)


def test_bad_block_table_entry_sets_status():
    w = W.make_workload(2, 16, [200, 300], paged=True, seed=14)
    w.block_table[1, 2] = 10 ** 6          # far outside the pool
    w.block_table[0, 0] = -5
    _, _, st, _ = run_cuda(w)
    assert st == -7


# ---------------------------------------------------------------- full-size workloads (sampled)
def _full(w, sample):
    o, lse, st, _ = run_cuda(w, poison=True)
    assert st == 0
    assert not np.isnan(o).any()
    o_ref, lse_ref = run_oracle(w, sample)
    return assert_parity(o[sample], lse[sample], o_ref, lse_ref, what="full-size sample")


def test_full_b16_h16_64k_sampled():
    w = W.workload_b16_h16(65536, seed=0, device="cuda")
    _full(w, [0, 11])


@pytest.mark.parametrize("L", [4096, 16384, 32768])
def test_full_b16_h16_sweep_sampled(L):
    w = W.workload_b16_h16(L, seed=0, device="cuda")
    _full(w, [3])


def test_full_b64_h16_paged_sampled():
    w = W.workload_b64_h16_paged(seed=0, device="cuda")
    lens = w.seqlens.tolist()
    sample = [int(np.argmin(lens)), int(np.argmax(lens)), 17]
    _full(w, sample)


def test_full_b32_h128_paged_sampled():
    w = W.workload_b32_h128_paged(seed=0, device="cuda")
    _full(w, [5])


def test_full_b16_h16_q4_causal_sampled():
    w = W.workload_b16_h16_q4_causal(seed=0, device="cuda")
    _full(w, [0, 9])


def test_bounded_waits_report_timeout_and_context_survives():
    """Failure detection without a GPU fault: with Q withheld the kernel's bounded waits
    run out (100 ms), it records MLA_ERR_TIMEOUT and returns; the next call is correct."""
    from mla_decode_attention_etap_b200 import FLAG_TEST_EXPIRE_WAITS
    w = W.make_workload(2, 16, [3000, 700], seed=15)
    _, _, st, dec = run_cuda(w, flags=FLAG_TEST_EXPIRE_WAITS, poison=False)
    assert st == -6  # MLA_ERR_TIMEOUT
    o, lse, st2, _ = run_cuda(w, decoder=dec)
    assert st2 == 0
    assert_parity(o, lse, *run_oracle(w), what="after an expired wait")
    w2 = W.make_workload(1, 128, [500], seed=16)
    _, _, st3, _ = run_cuda(w2, flags=FLAG_TEST_EXPIRE_WAITS, poison=False)
    assert st3 == -6


@pytest.mark.parametrize("heads", [16, 128])
def test_in_kernel_merge_matches_combine_and_resets_counters(heads):
    """The fused call merges split-KV partials itself (h = 16: the last split CTA of a sequence in
    the decode kernel; h = 128: the combine kernel started on the SMs the decode leaves, waiting on
    per-sequence split counters): bitwise equal to decode-with-partials + the separate combine
    kernel, including empty sequences, and repeatable without a new plan, before and after a
    call that skipped the merge (the counters rearm themselves)."""
    from mla_decode_attention_etap_b200 import FLAG_SKIP_COMBINE, mla_combine
    lens = [0, 5000, 1, 2900, 0, 777]
    w = W.make_workload(len(lens), heads, lens, seed=17, paged=heads == 128)
    dev = torch.device("cuda")
    q, kv, sl = w.q.to(dev), w.kv.to(dev), w.seqlens.to(dev)
    bt = w.block_table.to(dev) if w.block_table is not None else None
    from mla_decode_attention_etap_b200 import MlaDecoder
    dec = MlaDecoder(w.batch, w.q_len, w.num_heads, device=dev)
    shape = (w.batch, w.q_len, w.num_heads)
    outs = []
    dec.plan(sl)
    for _ in range(3):  # one plan, three fused calls
        o = torch.full(shape + (512,), float("nan"), dtype=torch.bfloat16, device=dev)
        lse = torch.full(shape, float("nan"), dtype=torch.float32, device=dev)
        dec.fwd(q, kv, sl, bt, w.softmax_scale, w.causal, o=o, lse=lse)
        outs.append((o.float().cpu().numpy(), lse.cpu().numpy()))
    torch.cuda.synchronize()
    assert dec.status() == 0
    o_s = torch.full(shape + (512,), float("nan"), dtype=torch.bfloat16, device=dev)
    l_s = torch.full(shape, float("nan"), dtype=torch.float32, device=dev)
    dec.fwd(q, kv, sl, bt, w.softmax_scale, w.causal, o=o_s, lse=l_s, flags=FLAG_SKIP_COMBINE)
    mla_combine(dec.workspace, w.batch, w.q_len, w.num_heads, dec.n_sms, o_s, l_s)
    for _ in range(2):  # fused calls again after the split path
        o = torch.full(shape + (512,), float("nan"), dtype=torch.bfloat16, device=dev)
        lse = torch.full(shape, float("nan"), dtype=torch.float32, device=dev)
        dec.fwd(q, kv, sl, bt, w.softmax_scale, w.causal, o=o, lse=lse)
        outs.append((o.float().cpu().numpy(), lse.cpu().numpy()))
    torch.cuda.synchronize()
    assert dec.status() == 0
    for o, l in outs:
        np.testing.assert_array_equal(o, o_s.float().cpu().numpy())
        np.testing.assert_array_equal(l, l_s.cpu().numpy())
    assert_parity(outs[0][0], outs[0][1], *run_oracle(w), what=f"in-kernel merge h={heads}")


def _a256(x):
    return (x + 255) & ~255


def _sched_offsets(off, batch, ctas_max, groups_max):
    """Byte offsets of one schedule's tables in the workspace (the layout of plan_core.h)."""
    t = {"ranges": off}
    off += _a256(4 * 2 * ctas_max)
    t["seq"] = off
    off += _a256(4 * ctas_max)
    t["tile"] = off
    off += _a256(4 * (batch + 1))
    t["info"] = off
    off += _a256(4 * 4 * batch)
    t["counters"] = off
    off += _a256(4 * 2 * batch * groups_max)
    t["done"] = off
    off += _a256(4 * batch)
    return t, off


@pytest.mark.parametrize("batch", [1, 7, 1024, 1500, 5000])
@pytest.mark.parametrize("heads", [16, 128])
def test_device_plan_matches_host_plan(batch, heads):
    """The block-scan plan kernel writes the same schedules as the host mirror (ranges, per-
    sequence units / first unit / splits / slot offsets, unit offsets, the grouping the M = 256
    kernel takes), for batches that give each plan thread zero, one or several sequences, with
    empty sequences mixed in."""
    from mla_decode_attention_etap_b200 import MlaDecoder, mla_decode_plan_host
    rng = np.random.default_rng(batch + heads)
    lens = rng.integers(0, 3000, size=batch).astype(np.int32)
    lens[rng.random(batch) < 0.2] = 0
    if heads == 128 and batch % 2:  # every nonempty sequence long: one 128-column group
        lens = np.where(lens > 0, lens + 8192, 0).astype(np.int32)
    dev = torch.device("cuda")
    dec = MlaDecoder(batch, 1, heads, device=dev)
    dec.plan(torch.tensor(lens, device=dev))
    torch.cuda.synchronize()
    ws = dec.workspace.view(torch.int32).cpu().numpy()
    ncols = heads
    n_sms = dec.n_sms
    # sizing of the two schedules (plan_core.h ws_layout)
    pair_groups = 1 if ncols <= 16 else (ncols + 31) // 32
    pair_ctas = max(1, n_sms // 2 // pair_groups)
    tabs = {}
    tabs[0], off = _sched_offsets(_a256(4 * 64), batch, pair_ctas, pair_groups)
    if ncols > 16:
        g0 = (ncols + 63) // 64
        c_max = max(1, n_sms // 2 // ((ncols + 127) // 128 if ncols > 64 else g0))
        tabs[1], off = _sched_offsets(off, batch, c_max, g0)
    for schedule, hdr in ((0, 8), (1, 16)):
        if schedule == 1 and ncols <= 16:
            continue
        ranges, info, nct, ngr, rows, gcols = mla_decode_plan_host(lens, 1, heads, n_sms, schedule)
        t = tabs[schedule]
        np.testing.assert_array_equal(ws[t["ranges"] // 4: t["ranges"] // 4 + 2 * nct].reshape(-1, 2), ranges)
        np.testing.assert_array_equal(ws[t["info"] // 4: t["info"] // 4 + 4 * batch].reshape(-1, 4), info)
        units = (lens.astype(np.int64) + rows - 1) // rows
        tile_off = np.concatenate([[0], np.cumsum(units)]).astype(np.int64)
        np.testing.assert_array_equal(ws[t["tile"] // 4: t["tile"] // 4 + batch + 1], tile_off.astype(np.int32))
        # each unit's first sequence: the one whose range holds the unit's first tile (batch if none)
        want = np.array([int(np.searchsorted(tile_off, fb, side="right") - 1) if fb < fe else batch
                         for fb, fe in ranges], dtype=np.int32)
        np.testing.assert_array_equal(ws[t["seq"] // 4: t["seq"] // 4 + nct], want)
        assert ws[hdr] == nct and ws[hdr + 1] == ngr and ws[hdr + 2] == int(units.sum()) and ws[hdr + 4] == gcols
    assert ws[0] == 0 and ws[1] == batch and ws[2] == ncols


@pytest.mark.parametrize("heads,q_len,causal", [(64, 1, False), (128, 2, False), (32, 4, True), (16, 8, True),
                                                (128, 8, True)])
def test_many_column_groups(heads, q_len, causal):
    """h*q_len from 64 to 1024 columns: 2..32 column groups of 32 (one cluster each per unit)."""
    w = W.make_workload(2, heads, [700, 130], q_len=q_len, causal=causal, seed=heads + q_len, paged=heads >= 128)
    o, lse, st, _ = run_cuda(w)
    assert st == 0
    assert_parity(o, lse, *run_oracle(w), what=f"h={heads} q={q_len}")


@pytest.mark.parametrize("heads,q_len,causal,paged", [(16, 1, False, False), (4, 4, True, False), (4, 4, False, True),
                                                      (16, 4, True, False), (16, 4, True, True), (32, 3, True, False)])
def test_ragged_q_lens(heads, q_len, causal, paged):
    """Ragged multi-token decode: per-sequence token counts 0..q_len (16- and 32-column groups)."""
    lens = [900, 3, 130, 257, 64]
    q_lens = [q_len, 0, 1, max(q_len - 1, 0), q_len]
    w = _poison_padding(W.make_workload(len(lens), heads, lens, q_len=q_len, causal=causal, paged=paged,
                                        seed=40 + heads + q_len, q_lens=q_lens, spike_frac=0.05))
    o, lse, st, _ = run_cuda(w)
    assert st == 0
    o_ref, lse_ref = run_oracle(w)
    for b, qb in enumerate(q_lens):          # padding tokens: exact zeros and -inf
        assert np.all(o[b, qb:] == 0) and np.all(np.isneginf(lse[b, qb:]))
    assert_parity(o, lse, o_ref, lse_ref, what=f"ragged h={heads} q={q_len}")


def test_ragged_q_lens_out_of_range_sets_status():
    w = W.make_workload(2, 16, [300, 200], q_len=2, seed=50, q_lens=[2, 1])
    w.q_lens[1] = 7                          # more tokens than q_len
    _, _, st, _ = run_cuda(w)
    assert st == -1                          # MLA_ERR_INVALID_ARG in the status word


def test_full_b16_h16_ragged_q4_causal_sampled():
    w = W.workload_b16_h16_ragged_q4_causal(seed=0, device="cuda")
    _full(w, [0, 5, 13])


def test_stream_probe_runs_clean():
    """The bandwidth probe (decode's TMA pattern without computation) completes with no expired wait."""
    import mla_decode_attention_etap_b200 as mla
    kv = torch.zeros(16 * 4096, 576, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for units in (74, 3):
        mla.mla_stream_probe(kv, units, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0


def test_cuda_graph_replay_matches_eager():
    """plan + fwd captured once in a CUDA graph (programmatic launches become graph edges) and
    replayed: bitwise the eager result, repeatedly (the merge counters reset themselves)."""
    from mla_decode_attention_etap_b200 import MlaDecoder
    w = W.make_workload(3, 16, [5000, 700, 2100], seed=60)
    dev = torch.device("cuda")
    q, kv, sl = w.q.to(dev), w.kv.to(dev), w.seqlens.to(dev)
    dec = MlaDecoder(w.batch, w.q_len, w.num_heads, device=dev)
    o = torch.empty(w.batch, 1, 16, 512, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(w.batch, 1, 16, dtype=torch.float32, device=dev)
    dec.plan(sl)
    dec.fwd(q, kv, sl, None, w.softmax_scale, False, o=o, lse=lse)
    torch.cuda.synchronize()
    o_eager, l_eager = o.clone(), lse.clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        o.zero_()
        with torch.cuda.graph(g, stream=side):
            dec.plan(sl, stream=side)
            dec.fwd(q, kv, sl, None, w.softmax_scale, False, o=o, lse=lse, stream=side)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(3):
        o.zero_()
        lse.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_eager) and torch.equal(lse, l_eager)
    assert dec.status() == 0


@pytest.mark.parametrize("q_len,lens", [(8, [700, 8]), (16, [1500, 40, 17]), (32, [2100, 333]), (64, [1000, 64, 65])])
def test_append_causal_moderate_q_len(q_len, lens):
    """Append attention: q_len = 8..64 new tokens per sequence, causal, 16 heads (N = 128..1024 query
    columns in groups of 32); includes caches barely longer than the appended tokens."""
    w = _poison_padding(W.make_workload(len(lens), 16, lens, q_len=q_len, causal=True, seed=70 + q_len,
                                        l_max=max(lens) + 50, spike_frac=0.02))
    o, lse, st, _ = run_cuda(w)
    assert st == 0
    assert_parity(o, lse, *run_oracle(w), what=f"append q_len={q_len}")


def test_append_ragged_paged():
    """Append with a different number of new tokens per sequence (0..16) on a paged cache."""
    lens = [900, 16, 1300, 5]
    q_lens = [16, 16, 3, 0]
    w = _poison_padding(W.make_workload(len(lens), 16, lens, q_len=16, causal=True, paged=True, seed=80,
                                        q_lens=q_lens))
    o, lse, st, _ = run_cuda(w)
    assert st == 0
    for b, qb in enumerate(q_lens):
        assert np.all(o[b, qb:] == 0) and np.all(np.isneginf(lse[b, qb:]))
    assert_parity(o, lse, *run_oracle(w), what="append ragged paged")


def test_full_b16_h16_append_q16_sampled():
    w = W.workload_b16_h16_append_q16(seed=0, device="cuda")
    _full(w, [0, 9])


@pytest.mark.parametrize("heads", [16, 64, 128])
def test_form_ablation_runs(heads):
    """The transposed/untransposed tensor-core ablation completes on every form and stream choice."""
    import mla_decode_attention_etap_b200 as mla
    dev = torch.device("cuda")
    cycles = torch.zeros(4, dtype=torch.int64, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for form in (0, 1):
        for streams in (1, 2, 3):
            cycles.zero_()
            mla.mla_form_ablation(form, heads, streams, 8, cycles, err)
            torch.cuda.synchronize()
            assert int(err.item()) == 0
            # at least 8 tiles x 16 MMAs at >= 8 cycles each
            assert int(cycles.min().item()) > 8 * 16 * 8


@pytest.mark.parametrize("heads,q_len,causal,lens", [(16, 1, False, [6000, 3000, 9000, 500]),
                                                     (16, 4, True, [3000, 2000, 700, 4100]),
                                                     (128, 1, False, [2500, 900])])
def test_repeated_decodes_are_bitwise_identical(heads, q_len, causal, lens):
    """Stress of the cross-CTA hand-offs (score exchange, slot release, pair merge): 200 plan +
    decode calls on one input must all give the bits of the first; a torn exchange would show up
    as a one-off difference.  The first result is also checked against the oracle."""
    from mla_decode_attention_etap_b200 import MlaDecoder
    w = W.make_workload(len(lens), heads, lens, q_len=q_len, causal=causal, seed=90 + heads + q_len)
    dev = torch.device("cuda")
    q, kv, sl = w.q.to(dev), w.kv.to(dev), w.seqlens.to(dev)
    dec = MlaDecoder(w.batch, w.q_len, w.num_heads, device=dev)
    o0 = lse0 = None
    bad = 0
    for i in range(200):
        dec.plan(sl)
        o, lse = dec.fwd(q, kv, sl, None, w.softmax_scale, w.causal)
        if o0 is None:
            o0, lse0 = o.clone(), lse.clone()
        elif not (torch.equal(o.view(torch.int16), o0.view(torch.int16)) and
                  torch.equal(lse.view(torch.int32), lse0.view(torch.int32))):
            bad += 1
    torch.cuda.synchronize()
    assert dec.status() == 0
    assert bad == 0, f"{bad} of 199 repeats differ from the first"
    assert_parity(o0.float().cpu().numpy(), lse0.cpu().numpy(), *run_oracle(w), what="repeat stress")
