"""Python binding of libmla_decode.so: MLA decode attention in the ETAP form on B200.

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  torch tensors provide device memory and the current stream.
The names mirror the C ABI in ``include/mla_decode.h``.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_decode.so")

D_QK = 576
D_V = 512
PAGE_SIZE = 64
FLAG_SKIP_COMBINE = 1
FLAG_TEST_EXPIRE_WAITS = 0x40000000

STATUS = {0: "MLA_OK", -1: "MLA_ERR_INVALID_ARG", -2: "MLA_ERR_UNSUPPORTED", -3: "MLA_ERR_ALIGNMENT",
          -4: "MLA_ERR_WORKSPACE", -5: "MLA_ERR_CUDA", -6: "MLA_ERR_TIMEOUT", -7: "MLA_ERR_BLOCK_TABLE"}

EXPORTS = ("mla_decode_workspace_size", "mla_decode_plan", "mla_decode_fwd", "mla_combine",
           "mla_decode_read_status", "mla_decode_plan_host", "mla_status_string", "mla_last_cuda_error",
           "mla_decode_fwd_static_ws", "mla_decode_static_ws_status", "mla_decode_fwd_ragged", "mla_stream_probe", "mla_decode_fwd_fp8", "mla_form_ablation",
           "mla_decode_fwd_trace", "mla_decode_fwd_untransposed")
STATIC_WORKSPACE_BYTES = 16777216


class MlaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)}")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library.  Raises if it was not built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m mla_decode_attention_etap_b200.build` "
                              "(or __graft_entry__.build()) first; there is no non-CUDA fallback")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        L.mla_decode_workspace_size.argtypes = [i32, i32, i32, i32]
        L.mla_decode_workspace_size.restype = sz
        L.mla_decode_plan.argtypes = [vp, i32, i32, i32, i32, vp, sz, vp]
        L.mla_decode_plan.restype = i32
        L.mla_decode_fwd.argtypes = [vp, vp, vp, vp, i32, i32, i32, i64, i32, ctypes.c_float, i32, vp, vp, vp, sz,
                                     i32, ctypes.c_uint, vp]
        L.mla_decode_fwd.restype = i32
        L.mla_decode_fwd_ragged.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i64, i32, ctypes.c_float, i32, vp, vp,
                                            vp, sz, i32, ctypes.c_uint, vp]
        L.mla_decode_fwd_ragged.restype = i32
        L.mla_decode_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i64, i32, ctypes.c_float, i32, vp,
                                         vp, vp, sz, i32, ctypes.c_uint, vp]
        L.mla_decode_fwd_fp8.restype = i32
        L.mla_decode_fwd_untransposed.argtypes = [vp, vp, vp, vp, i32, i32, i32, i64, i32, ctypes.c_float, i32, vp,
                                                  vp, vp, sz, i32, ctypes.c_uint, vp]
        L.mla_decode_fwd_untransposed.restype = i32
        L.mla_combine.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp]
        L.mla_combine.restype = i32
        L.mla_decode_read_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int), vp]
        L.mla_decode_read_status.restype = i32
        ip = ctypes.POINTER(ctypes.c_int)
        L.mla_decode_plan_host.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp, ip, ip, ip, ip]
        L.mla_decode_plan_host.restype = i32
        L.mla_status_string.argtypes = [i32]
        L.mla_status_string.restype = ctypes.c_char_p
        L.mla_decode_fwd_static_ws.argtypes = [vp, vp, vp, vp, i32, i32, i32, i64, i32, ctypes.c_float, i32, vp,
                                               vp, i32, vp]
        L.mla_decode_fwd_static_ws.restype = i32
        L.mla_decode_static_ws_status.argtypes = [ctypes.POINTER(ctypes.c_int), vp]
        L.mla_decode_static_ws_status.restype = i32
        L.mla_form_ablation.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp]
        L.mla_form_ablation.restype = i32
        L.mla_decode_fwd_trace.argtypes = [vp, vp, vp, vp, i32, i32, i32, i64, i32, ctypes.c_float, i32, vp, vp, vp,
                                           sz, i32, vp, i32, vp]
        L.mla_decode_fwd_trace.restype = i32
        L.mla_stream_probe.argtypes = [vp, i64, i32, vp, vp]
        L.mla_stream_probe.restype = i32
        L.mla_last_cuda_error.argtypes = []
        L.mla_last_cuda_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(code: int, what: str):
    if code != 0:
        if code == -5:
            what = f"{what} ({lib().mla_last_cuda_error().decode()})"
        raise MlaError(code, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _require(t, name: str, dtype, device, min_numel: int = 0, dim: Optional[int] = None,
             last: Optional[int] = None, min_rows: int = 0) -> None:
    """Reject a tensor whose raw pointer the library could not use safely: the C ABI sees only the
    pointer, so dtype, device, layout and size are checked here (TypeError / ValueError)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device} (all tensors on the device of q)")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name}: {t.dim()}-D, expected {dim}-D")
    if last is not None and (t.dim() == 0 or t.shape[-1] != last):
        raise ValueError(f"{name}: last dimension must be {last}, got shape {tuple(t.shape)}")
    if min_rows and (t.dim() == 0 or t.shape[0] < min_rows):
        raise ValueError(f"{name}: needs at least {min_rows} rows in dimension 0, got shape {tuple(t.shape)}")
    if t.numel() < min_numel:
        raise ValueError(f"{name}: {t.numel()} elements, needs at least {min_numel}")


def check_decode_args(q, kv, seqlens, block_table, o, lse, workspace, q_lens=None, kv_scale=None) -> None:
    """Shapes, dtypes and devices of a decode call (``kv_scale`` given: the FP8 cache, ``kv`` uint8)."""
    if not isinstance(q, torch.Tensor):
        raise TypeError("q: expected a torch.Tensor")
    dev = q.device
    _require(q, "q", torch.bfloat16, dev, dim=4, last=D_QK)
    B, q_len, h, _ = q.shape
    fp8 = kv_scale is not None
    _require(kv, "kv8" if fp8 else "kv", torch.uint8 if fp8 else torch.bfloat16, dev, dim=3, last=D_QK,
             min_rows=0 if block_table is not None else B)
    _require(seqlens, "seqlens", torch.int32, dev, min_numel=B, dim=1)
    if block_table is not None:
        _require(block_table, "block_table", torch.int32, dev, dim=2, min_rows=B)
    if q_lens is not None:
        _require(q_lens, "q_lens", torch.int32, dev, min_numel=B, dim=1)
    if fp8:
        _require(kv_scale, "kv_scale", torch.float32, dev, min_numel=kv.shape[0] * kv.shape[1])
    _require(o, "o", torch.bfloat16, dev, min_numel=B * q_len * h * D_V)
    _require(lse, "lse", torch.float32, dev, min_numel=B * q_len * h)
    _require(workspace, "workspace", None, dev)


def _require_cuda(t, name: str) -> None:
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor")


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def num_sms(device=None) -> int:
    return torch.cuda.get_device_properties(device if device is not None else torch.cuda.current_device()
                                            ).multi_processor_count


def mla_decode_workspace_size(batch: int, q_len: int, num_heads: int, n_sms: int) -> int:
    n = lib().mla_decode_workspace_size(batch, q_len, num_heads, n_sms)
    if n == 0:
        raise MlaError(-1, "mla_decode_workspace_size")
    return int(n)


def mla_decode_plan(seqlens: torch.Tensor, q_len: int, num_heads: int, workspace: torch.Tensor, n_sms: int,
                    stream=None) -> None:
    _require_cuda(seqlens, "seqlens")
    _require(seqlens, "seqlens", torch.int32, seqlens.device, dim=1)
    _require(workspace, "workspace", None, seqlens.device)
    _check(lib().mla_decode_plan(_ptr(seqlens), seqlens.numel(), q_len, num_heads, n_sms, _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)), "mla_decode_plan")


def mla_decode_fwd(q, kv, seqlens, block_table, softmax_scale, causal, o, lse, workspace, n_sms, flags=0,
                   stream=None, q_lens=None) -> None:
    """``q_lens`` (optional int32 device tensor [B]): ragged batch, q_lens[b] real query tokens of the
    q_len rows of sequence b (``mla_decode_fwd_ragged``)."""
    _require_cuda(q, "q")
    check_decode_args(q, kv, seqlens, block_table, o, lse, workspace, q_lens)
    B, q_len, h, _ = q.shape
    if block_table is not None:
        kv_rows, max_blocks = kv.shape[0] * kv.shape[1], block_table.shape[1]
    else:
        kv_rows, max_blocks = kv.shape[1], 0
    if q_lens is None:
        _check(lib().mla_decode_fwd(_ptr(q), _ptr(kv), _ptr(seqlens), _ptr(block_table), B, q_len, h, kv_rows,
                                    max_blocks, float(softmax_scale), int(bool(causal)), _ptr(o), _ptr(lse),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(), n_sms, flags,
                                    _stream(stream)), "mla_decode_fwd")
    else:
        _check(lib().mla_decode_fwd_ragged(_ptr(q), _ptr(kv), _ptr(seqlens), _ptr(q_lens), _ptr(block_table), B,
                                           q_len, h, kv_rows, max_blocks, float(softmax_scale), int(bool(causal)),
                                           _ptr(o), _ptr(lse), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(), n_sms, flags,
                                           _stream(stream)), "mla_decode_fwd_ragged")


def mla_decode_fwd_untransposed(q, kv, seqlens, block_table, softmax_scale, causal, o, lse, workspace, n_sms,
                                flags=0, stream=None) -> None:
    """The same decode in the untransposed form, S = Q K^T with the query columns on M (padded to 64
    or 128): the form the pages set ETAP against, for the A/B comparison (``mla_decode_fwd_untransposed``;
    bf16 cache, one q_len for every sequence)."""
    _require_cuda(q, "q")
    check_decode_args(q, kv, seqlens, block_table, o, lse, workspace)
    B, q_len, h, _ = q.shape
    if block_table is not None:
        kv_rows, max_blocks = kv.shape[0] * kv.shape[1], block_table.shape[1]
    else:
        kv_rows, max_blocks = kv.shape[1], 0
    _check(lib().mla_decode_fwd_untransposed(_ptr(q), _ptr(kv), _ptr(seqlens), _ptr(block_table), B, q_len, h,
                                             kv_rows, max_blocks, float(softmax_scale), int(bool(causal)), _ptr(o),
                                             _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                             n_sms, flags, _stream(stream)), "mla_decode_fwd_untransposed")


def mla_decode_fwd_fp8(q, kv8, kv_scale, seqlens, block_table, softmax_scale, causal, o, lse, workspace, n_sms,
                       flags=0, stream=None, q_lens=None) -> None:
    """Decode over an FP8 cache: ``kv8`` uint8 E4M3 codes laid out like the bf16 cache, ``kv_scale``
    fp32 with one scale per cache row (``mla_decode_fwd_fp8``; up to MLA_MAX_COLUMNS query columns)."""
    _require_cuda(q, "q")
    check_decode_args(q, kv8, seqlens, block_table, o, lse, workspace, q_lens, kv_scale=kv_scale)
    B, q_len, h, _ = q.shape
    if block_table is not None:
        kv_rows, max_blocks = kv8.shape[0] * kv8.shape[1], block_table.shape[1]
    else:
        kv_rows, max_blocks = kv8.shape[1], 0
    _check(lib().mla_decode_fwd_fp8(_ptr(q), _ptr(kv8), _ptr(kv_scale), _ptr(seqlens), _ptr(q_lens),
                                    _ptr(block_table), B, q_len, h, kv_rows, max_blocks, float(softmax_scale),
                                    int(bool(causal)), _ptr(o), _ptr(lse), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), n_sms, flags, _stream(stream)),
           "mla_decode_fwd_fp8")


TRACE_ROLES = ("K-tile producer", "step-1 issuer", "value producer", "softmax", "step-3 issuer")


def mla_decode_fwd_trace(q, kv, seqlens, block_table, softmax_scale, causal, o, lse, workspace, n_sms, trace,
                         stream=None) -> None:
    """mla_decode_fwd that also records the event stamps of cluster 0's roles into ``trace`` (int64 device
    tensor of 2 * 5 * cap + 4 * n_sms elements, zeroed by the caller, made by trace_buffer()); see
    decode_trace_events() and decode_trace_spans()."""
    _require_cuda(q, "q")
    check_decode_args(q, kv, seqlens, block_table, o, lse, workspace)
    _require(trace, "trace", torch.int64, q.device, dim=1)
    cap = (trace.numel() - 4 * n_sms) // (2 * len(TRACE_ROLES))
    if cap < 1 or trace.numel() != 2 * len(TRACE_ROLES) * cap + 4 * n_sms:
        raise ValueError("trace: use trace_buffer(cap, n_sms)")
    B, q_len, h, _ = q.shape
    if block_table is not None:
        kv_rows, max_blocks = kv.shape[0] * kv.shape[1], block_table.shape[1]
    else:
        kv_rows, max_blocks = kv.shape[1], 0
    _check(lib().mla_decode_fwd_trace(_ptr(q), _ptr(kv), _ptr(seqlens), _ptr(block_table), B, q_len, h, kv_rows,
                                      max_blocks, float(softmax_scale), int(bool(causal)), _ptr(o), _ptr(lse),
                                      _ptr(workspace), workspace.numel() * workspace.element_size(), n_sms,
                                      _ptr(trace), cap, _stream(stream)), "mla_decode_fwd_trace")


def trace_buffer(cap: int, n_sms: int, device=None):
    """A zeroed trace buffer for mla_decode_fwd_trace: [2 CTAs][5 roles][cap] stamps, then [n_sms][4]."""
    return torch.zeros(2 * len(TRACE_ROLES) * cap + 4 * n_sms, dtype=torch.int64, device=device)


def decode_trace_spans(trace, n_sms: int):
    """Trace buffer -> [n_sms, 4] (entry, start of work, end of work, exit) ns of every CTA, relative to the
    earliest entry (rows of CTAs that did not run stay 0)."""
    import numpy as np
    t = np.asarray(trace.cpu() if isinstance(trace, torch.Tensor) else trace).astype(np.int64)
    sp = t[len(t) - 4 * n_sms:].reshape(n_sms, 4).copy()
    live = sp[:, 0] > 0
    if live.any():
        sp[live] -= sp[live, 0].min()
    return sp


def decode_trace_events(trace, n_sms: int = None):
    """Trace buffer -> list of (cta, role, code, index, t_ns) sorted by time (t relative to the first stamp)."""
    import numpy as np
    t = np.asarray(trace.cpu() if isinstance(trace, torch.Tensor) else trace).astype(np.uint64)
    if n_sms is not None:
        t = t[:len(t) - 4 * n_sms]
    t = t.reshape(2, len(TRACE_ROLES), -1)
    out = []
    for cta in range(t.shape[0]):
        for role in range(t.shape[1]):
            for w in t[cta, role]:
                w = int(w)
                if w == 0:
                    break
                out.append((cta, role, w >> 56, (w >> 40) & 0xFFFF, w & 0xFFFFFFFFFF))
    if not out:
        return out
    t0 = min(e[4] for e in out)
    out = [(c, r, k, i, ts - t0) for c, r, k, i, ts in out]
    return sorted(out, key=lambda e: e[4])


def mla_stream_probe(kv, units: int, err, stream=None) -> None:
    """Stream ``kv`` ([..., 576] bf16, rows a multiple of 128) with the decode's TMA read pattern and
    no computation (a bandwidth probe).  ``err``: int32 device tensor [1], zeroed by the caller."""
    _require_cuda(kv, "kv")
    _require(kv, "kv", torch.bfloat16, kv.device, last=D_QK)
    _require(err, "err", torch.int32, kv.device, min_numel=1)
    rows = kv.numel() // 576
    _check(lib().mla_stream_probe(_ptr(kv), rows, units, _ptr(err), _stream(stream)), "mla_stream_probe")


def mla_form_ablation(form: int, heads: int, streams: int, tiles: int, cycles, err, stream=None) -> None:
    """Tensor-core instructions of ``tiles`` KV tiles per CTA in the transposed (form 0) or untransposed
    (form 1) layout; ``cycles``: uint64-compatible int64 device tensor [ctas], ``err``: int32 [1] zeroed."""
    _require_cuda(cycles, "cycles")
    _require(cycles, "cycles", torch.int64, cycles.device, min_numel=1)
    _require(err, "err", torch.int32, cycles.device, min_numel=1)
    _check(lib().mla_form_ablation(form, heads, streams, tiles, cycles.numel(), _ptr(cycles), _ptr(err),
                                   _stream(stream)), "mla_form_ablation")


def mla_combine(workspace, batch, q_len, num_heads, n_sms, o, lse, stream=None) -> None:
    _require_cuda(o, "o")
    _require(o, "o", torch.bfloat16, o.device, min_numel=batch * q_len * num_heads * D_V)
    _require(lse, "lse", torch.float32, o.device, min_numel=batch * q_len * num_heads)
    _require(workspace, "workspace", None, o.device)
    _check(lib().mla_combine(_ptr(workspace), batch, q_len, num_heads, n_sms, _ptr(o), _ptr(lse), _stream(stream)),
           "mla_combine")


def mla_decode_read_status(workspace, stream=None) -> int:
    _require_cuda(workspace, "workspace")
    out = ctypes.c_int(0)
    _check(lib().mla_decode_read_status(_ptr(workspace), ctypes.byref(out), _stream(stream)),
           "mla_decode_read_status")
    return int(out.value)


def mla_decode_plan_host(seqlens, q_len: int, num_heads: int, n_sms: int, schedule: int = 1):
    """Host mirror of a schedule -> (cta_ranges [ctas, 2], seq_info [B, 4], num_ctas, num_groups, unit_rows,
    group_cols).  schedule 1: the one mla_decode_fwd (bf16 cache) uses; 0: the one mla_decode_fwd_fp8 uses."""
    import numpy as np
    sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    nct, ngr, urows, gcols = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().mla_decode_plan_host(sl.ctypes.data_as(ctypes.c_void_p), sl.size, q_len, num_heads, n_sms, schedule,
                                      None, None, ctypes.byref(nct), ctypes.byref(ngr), ctypes.byref(urows),
                                      ctypes.byref(gcols)), "mla_decode_plan_host")
    ranges = np.zeros((nct.value, 2), np.int32)
    info = np.zeros((sl.size, 4), np.int32)
    _check(lib().mla_decode_plan_host(sl.ctypes.data_as(ctypes.c_void_p), sl.size, q_len, num_heads, n_sms, schedule,
                                      ranges.ctypes.data_as(ctypes.c_void_p), info.ctypes.data_as(ctypes.c_void_p),
                                      ctypes.byref(nct), ctypes.byref(ngr), ctypes.byref(urows), ctypes.byref(gcols)),
           "mla_decode_plan_host")
    return ranges, info, nct.value, ngr.value, urows.value, gcols.value


class MlaDecoder:
    """Owns the workspace for one (batch, q_len, num_heads) shape; plan() then fwd()."""

    def __init__(self, batch: int, q_len: int, num_heads: int, device=None, n_sms: Optional[int] = None):
        self.device = torch.device(device if device is not None else "cuda")
        self.batch, self.q_len, self.num_heads = batch, q_len, num_heads
        self.n_sms = n_sms if n_sms is not None else num_sms(self.device)
        nbytes = mla_decode_workspace_size(batch, q_len, num_heads, self.n_sms)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)

    def plan(self, seqlens: torch.Tensor, stream=None):
        mla_decode_plan(seqlens, self.q_len, self.num_heads, self.workspace, self.n_sms, stream)

    def fwd(self, q, kv, seqlens, block_table=None, softmax_scale=None, causal=False, o=None, lse=None,
            flags=0, stream=None, q_lens=None):
        B, q_len, h, _ = q.shape
        if o is None:
            o = torch.empty(B, q_len, h, D_V, dtype=torch.bfloat16, device=q.device)
        if lse is None:
            lse = torch.empty(B, q_len, h, dtype=torch.float32, device=q.device)
        scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(D_QK)
        mla_decode_fwd(q, kv, seqlens, block_table, scale, causal, o, lse, self.workspace, self.n_sms, flags,
                       stream, q_lens=q_lens)
        return o, lse

    def fwd_fp8(self, q, kv8, kv_scale, seqlens, block_table=None, softmax_scale=None, causal=False, o=None,
                lse=None, flags=0, stream=None, q_lens=None):
        """fwd over an FP8 cache (E4M3 codes + one fp32 scale per cache row)."""
        B, q_len, h, _ = q.shape
        if o is None:
            o = torch.empty(B, q_len, h, D_V, dtype=torch.bfloat16, device=q.device)
        if lse is None:
            lse = torch.empty(B, q_len, h, dtype=torch.float32, device=q.device)
        scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(D_QK)
        mla_decode_fwd_fp8(q, kv8, kv_scale, seqlens, block_table, scale, causal, o, lse, self.workspace, self.n_sms,
                           flags, stream, q_lens=q_lens)
        return o, lse

    def status(self, stream=None) -> int:
        return mla_decode_read_status(self.workspace, stream)


def mla_decode(q, kv, seqlens, block_table=None, softmax_scale=None, causal=False, q_lens=None):
    """One-shot convenience: plan + decode (+ combine).  Returns (O bf16, LSE fp32)."""
    dec = MlaDecoder(q.shape[0], q.shape[1], q.shape[2], device=q.device)
    dec.plan(seqlens)
    return dec.fwd(q, kv, seqlens, block_table, softmax_scale, causal, q_lens=q_lens)
