"""TEST INFRASTRUCTURE — Python front end of the fp64 MLA decode oracle.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
use this module.  It never imports the CUDA package: callers hand it arrays
(bf16 passed as uint16 bit patterns).

Two independent fp64 implementations of the same definition live here:

* ``mla_decode`` / ``mla_decode_etap`` — the C oracle (``mla_oracle.c``), in the
  standard form S = Q K^T, P = softmax(S), O = P V and in the transposed ETAP
  form S^T = K Q^T, P^T = softmax(S^T), O^T = V^T P^T, O = (O^T)^T
  (FlashMLA-ETAP technical summary, "Methodology", the ETAP step list);
* ``mla_decode_numpy`` — the standard form written with numpy fp64 matmuls, used
  to cross-check the C code.

``lse_merge`` is the log-sum-exp merge of results over disjoint KV ranges.

``mla_decode_fp8`` / ``mla_decode_fp8_numpy`` take an FP8 latent cache (an
adjacent storage format, not on the pages): E4M3 codes (uint8) plus one fp32
scale per cache row; element k of row r is scale[r] * e4m3(code[r, k]), and
the attention is the same definition on those widened values.
"""

from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional

import numpy as np

D_QK = 576
D_V = 512
PAGE = 64

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_LIB = os.path.join(_HERE, "libmla_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, OpenMP) next to its source; returns the .so path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        args = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
                ctypes.c_void_p, ctypes.c_void_p]
        for name in ("oracle_mla_decode", "oracle_mla_decode_etap"):
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        lib.oracle_mla_decode_ragged.argtypes = args[:3] + [ctypes.c_void_p] + args[3:]
        lib.oracle_mla_decode_ragged.restype = ctypes.c_int
        lib.oracle_mla_decode_fp8.argtypes = ([ctypes.c_void_p] * 6 + [ctypes.c_int] * 8 +
                                              [ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p])
        lib.oracle_mla_decode_fp8.restype = ctypes.c_int
        lib.oracle_lse_merge.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_lse_merge.restype = None
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _call(name, q_bits, kv_bits, seqlens, block_table, scale, causal, threads=None, q_lens=None):
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    kv_bits = np.ascontiguousarray(kv_bits, dtype=np.uint16)
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    B, q_len, h, dqk = q_bits.shape
    assert dqk == D_QK and kv_bits.shape[-1] == D_QK
    if block_table is not None:
        block_table = np.ascontiguousarray(block_table, dtype=np.int32)
        kv_rows, max_blocks, page = 0, block_table.shape[1], kv_bits.shape[1]
    else:
        kv_rows, max_blocks, page = kv_bits.shape[1], 0, PAGE
    o = np.zeros((B, q_len, h, D_V), dtype=np.float64)
    lse = np.zeros((B, q_len, h), dtype=np.float64)
    if threads is not None:
        os.environ["OMP_NUM_THREADS"] = str(threads)
    if q_lens is None:
        rc = getattr(_load(), name)(_ptr(q_bits), _ptr(kv_bits), _ptr(seqlens), _ptr(block_table),
                                    B, q_len, h, D_QK, D_V, kv_rows, max_blocks, page,
                                    float(scale), int(bool(causal)), _ptr(o), _ptr(lse))
    else:
        q_lens = np.ascontiguousarray(q_lens, dtype=np.int32)
        assert q_lens.shape == (B,) and q_lens.min() >= 0 and q_lens.max() <= q_len
        rc = _load().oracle_mla_decode_ragged(_ptr(q_bits), _ptr(kv_bits), _ptr(seqlens), _ptr(q_lens),
                                              _ptr(block_table), B, q_len, h, D_QK, D_V, kv_rows, max_blocks,
                                              page, float(scale), int(bool(causal)), _ptr(o), _ptr(lse))
    if rc != 0:
        raise MemoryError(f"{name} failed ({rc})")
    return o, lse


def mla_decode(q_bits, kv_bits, seqlens, block_table=None, scale=1.0 / 24.0, causal=False, q_lens=None):
    """Standard-form oracle.  Returns (O fp64 [B,q,h,512], LSE fp64 [B,q,h]).

    ``q_lens`` (optional, [B]): ragged multi-token decode, q_lens[b] real query tokens in
    sequence b (the rest of the q_len positions are padding: O = 0, LSE = -inf)."""
    return _call("oracle_mla_decode", q_bits, kv_bits, seqlens, block_table, scale, causal, q_lens=q_lens)


def mla_decode_etap(q_bits, kv_bits, seqlens, block_table=None, scale=1.0 / 24.0, causal=False):
    """Transposed-form (ETAP steps 1-4) oracle.  Same outputs as ``mla_decode``."""
    return _call("oracle_mla_decode_etap", q_bits, kv_bits, seqlens, block_table, scale, causal)


def mla_decode_fp8(q_bits, kv_codes, kv_scale, seqlens, block_table=None, scale=1.0 / 24.0, causal=False,
                   q_lens=None, threads=None):
    """Standard-form oracle on an FP8 cache: ``kv_codes`` uint8 E4M3 codes laid out like the bf16
    cache, ``kv_scale`` fp32 with one scale per cache row ([B, kv_rows] or [num_blocks, 64]).
    Returns (O fp64 [B,q,h,512], LSE fp64 [B,q,h])."""
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    kv_codes = np.ascontiguousarray(kv_codes, dtype=np.uint8)
    kv_scale = np.ascontiguousarray(kv_scale, dtype=np.float32)
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    B, q_len, h, dqk = q_bits.shape
    assert dqk == D_QK and kv_codes.shape[-1] == D_QK and kv_scale.shape == kv_codes.shape[:-1]
    if block_table is not None:
        block_table = np.ascontiguousarray(block_table, dtype=np.int32)
        kv_rows, max_blocks, page = 0, block_table.shape[1], kv_codes.shape[1]
    else:
        kv_rows, max_blocks, page = kv_codes.shape[1], 0, PAGE
    if q_lens is not None:
        q_lens = np.ascontiguousarray(q_lens, dtype=np.int32)
        assert q_lens.shape == (B,) and q_lens.min() >= 0 and q_lens.max() <= q_len
    o = np.zeros((B, q_len, h, D_V), dtype=np.float64)
    lse = np.zeros((B, q_len, h), dtype=np.float64)
    if threads is not None:
        os.environ["OMP_NUM_THREADS"] = str(threads)
    rc = _load().oracle_mla_decode_fp8(_ptr(q_bits), _ptr(kv_codes), _ptr(kv_scale), _ptr(seqlens), _ptr(q_lens),
                                       _ptr(block_table), B, q_len, h, D_QK, D_V, kv_rows, max_blocks, page,
                                       float(scale), int(bool(causal)), _ptr(o), _ptr(lse))
    if rc != 0:
        raise MemoryError(f"oracle_mla_decode_fp8 failed ({rc})")
    return o, lse


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """OCP E4M3 codes -> fp64: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is
    subnormal, 0x7F / 0xFF are NaN, there are no infinities."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e, m = (c >> 3) & 15, c & 7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(c & 0x80, -mag, mag)


def mla_decode_fp8_numpy(q_bits, kv_codes, kv_scale, seqlens, block_table=None, scale=1.0 / 24.0, causal=False,
                         q_lens=None):
    """Second, independent fp64 implementation on the FP8 cache (numpy matmuls on the widened rows)."""
    kv = e4m3_to_f64(kv_codes) * np.asarray(kv_scale, dtype=np.float64)[..., None]
    return _decode_numpy_f64(bf16_bits_to_f64(q_bits), kv, seqlens, block_table, scale, causal, q_lens)


def lse_merge(o_s: np.ndarray, lse_s: np.ndarray):
    """Merge S partial results over disjoint KV ranges: o_s [S, d], lse_s [S] -> (o [d], lse)."""
    o_s = np.ascontiguousarray(o_s, dtype=np.float64)
    lse_s = np.ascontiguousarray(lse_s, dtype=np.float64)
    S, d = o_s.shape
    o = np.zeros(d, dtype=np.float64)
    lse = np.zeros(1, dtype=np.float64)
    _load().oracle_lse_merge(S, d, _ptr(o_s), _ptr(lse_s), _ptr(o), _ptr(lse))
    return o, float(lse[0])


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp64."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (nearest-even via fp32), returning bit patterns; for building test inputs."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def mla_decode_numpy(q_bits, kv_bits, seqlens, block_table=None, scale=1.0 / 24.0, causal=False, q_lens=None):
    """Second, independent fp64 implementation of the standard form with numpy matmuls."""
    return _decode_numpy_f64(bf16_bits_to_f64(q_bits), bf16_bits_to_f64(kv_bits), seqlens, block_table, scale,
                             causal, q_lens)


def _decode_numpy_f64(q, kv, seqlens, block_table, scale, causal, q_lens):
    B, q_len, h, _ = q.shape
    o = np.zeros((B, q_len, h, D_V))
    lse = np.zeros((B, q_len, h))
    for b in range(B):
        L = int(seqlens[b])
        if block_table is not None:
            page = kv.shape[1]
            nb = (L + page - 1) // page
            rows = kv[np.asarray(block_table[b, :nb], dtype=np.int64)].reshape(nb * page, D_QK)[:L]
        else:
            rows = kv[b, :L]
        qb = q_len if q_lens is None else int(q_lens[b])
        for t in range(q_len):
            if t >= qb:
                vis = 0                                   # padding token of a ragged batch
            else:
                vis = max(L - qb + t + 1, 0) if causal else L
            if vis == 0:
                lse[b, t] = -math.inf
                continue
            S = scale * (q[b, t] @ rows[:vis].T)          # [h, vis]
            m = S.max(axis=1, keepdims=True)
            E = np.exp(S - m)
            den = E.sum(axis=1, keepdims=True)
            o[b, t] = (E / den) @ rows[:vis, :D_V]
            lse[b, t] = (m + np.log(den))[:, 0]
    return o, lse
