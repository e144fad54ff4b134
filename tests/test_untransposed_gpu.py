"""GPU parity of the untransposed form (S = Q K^T, heads on the MMA's M, padded to 64 / 128) against
the fp64 oracle: the second arm of the transposed-vs-untransposed comparison, held to the same bar
as the ETAP kernels (tests/parity.py) on the same seeded inputs."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import mla_decode_attention_etap_b200 as mla
from mla_decode_attention_etap_b200 import workloads as W
from tests.parity import assert_parity, run_cuda, run_oracle
from tests.test_parity_gpu import _poison_padding

pytestmark = pytest.mark.gpu


def run_untransposed(w: W.Workload, n_sms=None):
    dev = torch.device("cuda")
    q, kv, sl = w.q.to(dev), w.kv.to(dev), w.seqlens.to(dev)
    bt = w.block_table.to(dev) if w.block_table is not None else None
    dec = mla.MlaDecoder(w.batch, w.q_len, w.num_heads, device=dev, n_sms=n_sms)
    o = torch.full((w.batch, w.q_len, w.num_heads, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((w.batch, w.q_len, w.num_heads), float("nan"), dtype=torch.float32, device=dev)
    dec.plan(sl)
    mla.mla_decode_fwd_untransposed(q, kv, sl, bt, w.softmax_scale, w.causal, o, lse, dec.workspace, dec.n_sms)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), lse.cpu().numpy(), dec.status()


def test_h16_edge_lengths_nan_padding():
    """16 heads padded to M = 64 on the 16-column schedule: tails, a one-row sequence, an empty one."""
    lens = [1, 63, 64, 65, 127, 128, 129, 1000, 0, 3000]
    w = _poison_padding(W.make_workload(len(lens), 16, lens, seed=31))
    o, lse, st = run_untransposed(w)
    assert st == 0
    o_ref, lse_ref = run_oracle(w)
    assert np.all(o[8] == 0) and np.all(np.isneginf(lse[8]))
    assert_parity(o, lse, o_ref, lse_ref, what="untransposed h=16")


@pytest.mark.parametrize("n_sms", [1, 7, 148, 600])
def test_h16_split_counts(n_sms):
    w = W.make_workload(3, 16, [3000, 257, 1536], seed=32)
    o, lse, st = run_untransposed(w, n_sms=n_sms)
    assert st == 0
    assert_parity(o, lse, *run_oracle(w), what=f"untransposed n_sms={n_sms}")


def test_q4_causal_spikes():
    """q_len = 4, causal, rows scaled x8: 64 query columns in one M = 64 group, rescales taken."""
    lens = [5, 130, 2000, 777]
    w = W.make_workload(len(lens), 16, lens, q_len=4, causal=True, seed=33, spike_frac=0.05, spike_scale=8.0)
    o, lse, st = run_untransposed(w)
    assert st == 0
    assert_parity(o, lse, *run_oracle(w), what="untransposed q4 causal")


def test_h128_paged_short():
    """128 heads, sequences under 8192 rows: two 64-column groups (M = 64, P as hi + lo)."""
    lens = [300, 4097, 0, 2500]
    w = _poison_padding(W.make_workload(len(lens), 128, lens, seed=34, paged=True))
    o, lse, st = run_untransposed(w)
    assert st == 0
    assert_parity(o, lse, *run_oracle(w), what="untransposed h=128 paged")


def test_h128_paged_long_single_group():
    """128 heads, every sequence >= 8192 rows: one 128-column group (M = 128, one bf16 P term),
    the configuration of the B=32 h=128 workload."""
    lens = [8192, 9001]
    w = W.make_workload(len(lens), 128, lens, seed=35, paged=True)
    o, lse, st = run_untransposed(w)
    assert st == 0
    assert_parity(o, lse, *run_oracle(w), what="untransposed h=128 one group")


def test_same_inputs_both_forms():
    """Both forms on the same inputs, both against the oracle (the comparison's precondition)."""
    lens = [2048, 64, 999]
    w = W.make_workload(len(lens), 16, lens, seed=36)
    o_ref, lse_ref = run_oracle(w)
    o_u, l_u, st_u = run_untransposed(w)
    o_t, l_t, st_t, _ = run_cuda(w)
    assert st_u == 0 and st_t == 0
    assert_parity(o_u, l_u, o_ref, lse_ref, what="untransposed")
    assert_parity(o_t, l_t, o_ref, lse_ref, what="transposed")


def test_full_b32_h128_paged_sampled():
    """The full B=32 h=128 paged workload in the bench's launch configuration (148 SMs), compared on
    sampled sequences the oracle computes one by one."""
    w = W.workload_b32_h128_paged(seed=0)
    o, lse, st = run_untransposed(w, n_sms=148)
    assert st == 0
    idx = [0, 13, 31]
    o_ref, lse_ref = run_oracle(w, batch_index=idx)
    assert_parity(o[idx], lse[idx], o_ref, lse_ref, what="untransposed B=32 h=128 sampled")
