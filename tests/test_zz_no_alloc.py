"""The entry point that allocates nothing (mla_decode_fwd_static_ws) and its status reader.

It serves callers that cannot allocate device memory: a plugin inside a host
framework that owns all GPU memory and offers no allocator, or a serving loop
that must not call cudaMalloc/cudaFree because they can synchronise the device.
Its scratch is a static device array inside the library, shared by every call.

The GPU tests call it through the C ABI twice in a row, on two different
batches.  Both calls run the same plan and decode kernels as the regular entry
point (mla_decode_plan + mla_decode_fwd with a caller-owned workspace) on the
same number of SMs, so their outputs must agree bit for bit; each result is
also checked against the fp64 oracle with the parity tolerance of the other
tests.  A bad block-table entry must surface as MLA_ERR_BLOCK_TABLE through
mla_decode_static_ws_status, and the next good call must clear it.  This file
is collected last on purpose.
"""

from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import mla_decode_attention_etap_b200 as mla
from mla_decode_attention_etap_b200 import workloads as W
from tests.parity import assert_parity, run_oracle


def _call_static(w, dev, n_sms):
    q, kv = w.q.to(dev), w.kv.to(dev)
    sl = w.seqlens.to(dev)
    bt = w.block_table.to(dev) if w.block_table is not None else None
    o = torch.full((w.batch, w.q_len, w.num_heads, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((w.batch, w.q_len, w.num_heads), float("nan"), dtype=torch.float32, device=dev)
    if bt is not None:
        kv_rows, max_blocks = kv.shape[0] * kv.shape[1], bt.shape[1]
    else:
        kv_rows, max_blocks = kv.shape[1], 0
    vp = ctypes.c_void_p
    rc = mla.lib().mla_decode_fwd_static_ws(
        vp(q.data_ptr()), vp(kv.data_ptr()), vp(sl.data_ptr()), vp(bt.data_ptr()) if bt is not None else None,
        w.batch, w.q_len, w.num_heads, kv_rows, max_blocks, ctypes.c_float(w.softmax_scale), int(w.causal),
        vp(o.data_ptr()), vp(lse.data_ptr()), n_sms, vp(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, mla.STATUS.get(rc, rc)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def _static_status():
    out = ctypes.c_int(12345)
    rc = mla.lib().mla_decode_static_ws_status(ctypes.byref(out),
                                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, mla.STATUS.get(rc, rc)
    return int(out.value)


def _call_regular(w, dev, n_sms):
    dec = mla.MlaDecoder(w.batch, w.q_len, w.num_heads, device=dev, n_sms=n_sms)
    sl = w.seqlens.to(dev)
    dec.plan(sl)
    o, lse = dec.fwd(w.q.to(dev), w.kv.to(dev), sl,
                     w.block_table.to(dev) if w.block_table is not None else None, w.softmax_scale, w.causal)
    torch.cuda.synchronize()
    assert dec.status() == 0
    return o.cpu(), lse.cpu()


@pytest.mark.gpu
def test_static_workspace_matches_regular_entry_point_twice():
    dev = torch.device("cuda")
    n_sms = mla.num_sms(dev)
    # first call: a long split batch; second call: a smaller paged causal multi-token batch that
    # reuses the same static scratch and must not see the first call's leftovers
    first = W.make_workload(4, 16, [9000, 300, 4096, 1], seed=21)
    second = W.make_workload(3, 16, [700, 64, 2500], q_len=4, causal=True, paged=True, seed=22)
    for w in (first, second):
        o_s, l_s = _call_static(w, dev, n_sms)
        assert _static_status() == 0
        o_r, l_r = _call_regular(w, dev, n_sms)
        # same kernels, same schedule: identical bits (NaN-poisoned outputs would show as holes)
        assert not torch.isnan(o_s.float()).any()
        np.testing.assert_array_equal(o_s.view(torch.int16).numpy(), o_r.view(torch.int16).numpy())
        np.testing.assert_array_equal(l_s.view(torch.int32).numpy(), l_r.view(torch.int32).numpy())
        o_ref, lse_ref = run_oracle(w)
        assert_parity(o_s.float().numpy(), l_s.numpy(), o_ref, lse_ref, what="static-workspace entry point")


@pytest.mark.gpu
def test_static_workspace_status_reports_bad_block_table_then_clears():
    dev = torch.device("cuda")
    n_sms = mla.num_sms(dev)
    bad = W.make_workload(2, 16, [200, 300], paged=True, seed=14)
    bad.block_table[1, 2] = 10 ** 6   # far outside the pool: never dereferenced, recorded in the status word
    bad.block_table[0, 0] = -5
    _call_static(bad, dev, n_sms)
    assert _static_status() == -7     # MLA_ERR_BLOCK_TABLE
    good = W.make_workload(2, 16, [200, 300], paged=True, seed=14)
    o, lse = _call_static(good, dev, n_sms)
    assert _static_status() == 0      # the next call's schedule rewrites the status word
    o_ref, lse_ref = run_oracle(good)
    assert_parity(o.float().numpy(), lse.numpy(), o_ref, lse_ref, what="static-workspace call after a bad one")


def test_static_workspace_rejects_shapes_beyond_its_size():
    """B=32, h=128 needs more scratch than the static array holds: refused before any launch."""
    A = ctypes.c_void_p(1 << 20)
    need = mla.mla_decode_workspace_size(32, 1, 128, 148)
    assert need > mla.STATIC_WORKSPACE_BYTES
    rc = mla.lib().mla_decode_fwd_static_ws(A, A, A, None, 32, 1, 128, 32768, 0, ctypes.c_float(1 / 24), 0, A, A,
                                            148, None)
    assert rc == -4  # MLA_ERR_WORKSPACE
    assert mla.mla_decode_workspace_size(16, 1, 16, 148) <= mla.STATIC_WORKSPACE_BYTES


def test_static_workspace_status_rejects_null():
    assert mla.lib().mla_decode_static_ws_status(None, None) == -1  # MLA_ERR_INVALID_ARG, nothing copied
