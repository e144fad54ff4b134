"""Shared helpers for the parity tests: run the CUDA path and the oracle on the same inputs."""

from __future__ import annotations

import math

import numpy as np
import torch

from mla_decode_attention_etap_b200 import MlaDecoder
from mla_decode_attention_etap_b200.workloads import Workload, bf16_bits
from oracle import mla_oracle as om

# Tolerances of the parity bar, applied to the whole compared tensor:
RMSE_REL = 2e-3     # RMSE(O - O_ref) <= 2e-3 * RMS(O_ref)
MAXABS_REL = 1e-2   # max|O - O_ref| <= 1e-2 * max|O_ref|
LSE_ABS = 1e-3      # max|LSE - LSE_ref| <= 1e-3 (natural log)


def run_cuda(w: Workload, n_sms=None, flags=0, poison=True, decoder=None):
    """Plan + decode (+ combine) through the C ABI; outputs pre-filled with NaN to catch holes."""
    dev = torch.device("cuda")
    q = w.q.to(dev)
    kv = w.kv.to(dev)
    sl = w.seqlens.to(dev)
    bt = w.block_table.to(dev) if w.block_table is not None else None
    dec = decoder or MlaDecoder(w.batch, w.q_len, w.num_heads, device=dev, n_sms=n_sms)
    o = torch.full((w.batch, w.q_len, w.num_heads, 512), float("nan") if poison else 0.0,
                   dtype=torch.bfloat16, device=dev)
    lse = torch.full((w.batch, w.q_len, w.num_heads), float("nan") if poison else 0.0,
                     dtype=torch.float32, device=dev)
    dec.plan(sl)
    ql = w.q_lens.to(dev) if w.q_lens is not None else None
    if w.fp8:
        dec.fwd_fp8(q, w.kv8.to(dev), w.kv_scale.to(dev), sl, bt, w.softmax_scale, w.causal, o=o, lse=lse,
                    flags=flags, q_lens=ql)
    else:
        dec.fwd(q, kv, sl, bt, w.softmax_scale, w.causal, o=o, lse=lse, flags=flags, q_lens=ql)
    torch.cuda.synchronize()
    status = dec.status()
    return o.float().cpu().numpy(), lse.cpu().numpy(), status, dec


def run_oracle(w: Workload, batch_index=None):
    """fp64 oracle on all sequences, or on the listed ones (each resolved to a contiguous copy)."""
    if w.fp8:
        return _run_oracle_fp8(w, batch_index)
    if batch_index is None:
        q = bf16_bits(w.q)
        kv = bf16_bits(w.kv)
        bt = None if w.block_table is None else w.block_table.numpy()
        ql = None if w.q_lens is None else w.q_lens.numpy()
        return om.mla_decode(q, kv, w.seqlens.numpy(), bt, w.softmax_scale, w.causal, q_lens=ql)
    outs_o, outs_l = [], []
    for b in batch_index:
        L = int(w.seqlens[b])
        rows = w.kv_rows(b).cpu()
        kv = bf16_bits(rows.reshape(1, max(L, 0), 576)) if L > 0 else np.zeros((1, 1, 576), np.uint16)
        q = bf16_bits(w.q[b:b + 1].cpu())
        ql = None if w.q_lens is None else w.q_lens[b:b + 1].numpy()
        o, lse = om.mla_decode(q, kv, np.array([L], np.int32), None, w.softmax_scale, w.causal, q_lens=ql)
        outs_o.append(o[0])
        outs_l.append(lse[0])
    return np.stack(outs_o), np.stack(outs_l)


def _seq_rows(w: Workload, t: torch.Tensor, b: int) -> torch.Tensor:
    """Logical rows [L_b, ...] of a per-row cache tensor (codes or scales) of sequence b."""
    L = int(w.seqlens[b])
    if w.block_table is None:
        return t[b, :L]
    nb = (L + 63) // 64
    return t[w.block_table[b, :nb].long()].reshape(nb * 64, *t.shape[2:])[:L]


def _run_oracle_fp8(w: Workload, batch_index):
    if batch_index is None:
        bt = None if w.block_table is None else w.block_table.numpy()
        ql = None if w.q_lens is None else w.q_lens.numpy()
        return om.mla_decode_fp8(bf16_bits(w.q), w.kv8.numpy(), w.kv_scale.numpy(), w.seqlens.numpy(), bt,
                                 w.softmax_scale, w.causal, q_lens=ql)
    outs_o, outs_l = [], []
    for b in batch_index:
        L = int(w.seqlens[b])
        codes = _seq_rows(w, w.kv8, b).numpy().reshape(1, L, 576) if L > 0 else np.zeros((1, 1, 576), np.uint8)
        sc = _seq_rows(w, w.kv_scale, b).numpy().reshape(1, L) if L > 0 else np.ones((1, 1), np.float32)
        ql = None if w.q_lens is None else w.q_lens[b:b + 1].numpy()
        o, lse = om.mla_decode_fp8(bf16_bits(w.q[b:b + 1].cpu()), codes, sc, np.array([L], np.int32), None,
                                   w.softmax_scale, w.causal, q_lens=ql)
        outs_o.append(o[0])
        outs_l.append(lse[0])
    return np.stack(outs_o), np.stack(outs_l)


def parity_metrics(o, lse, o_ref, lse_ref):
    o = np.asarray(o, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    err = o - o_ref
    rms_ref = math.sqrt(float(np.mean(o_ref ** 2))) if o_ref.size else 0.0
    rmse = math.sqrt(float(np.mean(err ** 2))) if err.size else 0.0
    finite = np.isfinite(lse_ref)
    lse_err = float(np.max(np.abs(lse[finite] - lse_ref[finite]))) if finite.any() else 0.0
    return {
        "rmse": rmse, "rms_ref": rms_ref, "rmse_rel": rmse / rms_ref if rms_ref > 0 else rmse,
        "maxabs": float(np.max(np.abs(err))) if err.size else 0.0,
        "max_ref": float(np.max(np.abs(o_ref))) if o_ref.size else 0.0,
        "lse_err": lse_err,
        "nan_o": int(np.isnan(o).sum()),
        "inf_lse_mismatch": int(np.sum(np.isneginf(lse_ref) != np.isneginf(lse))),
    }


def assert_parity(o, lse, o_ref, lse_ref, what=""):
    m = parity_metrics(o, lse, o_ref, lse_ref)
    assert m["nan_o"] == 0, f"{what}: {m['nan_o']} NaN outputs {m}"
    assert m["inf_lse_mismatch"] == 0, f"{what}: -inf LSE pattern differs {m}"
    assert m["rmse"] <= RMSE_REL * m["rms_ref"] + 1e-12, f"{what}: RMSE {m}"
    assert m["maxabs"] <= MAXABS_REL * m["max_ref"] + 1e-12, f"{what}: max-abs {m}"
    assert m["lse_err"] <= LSE_ABS, f"{what}: LSE {m}"
    return m
