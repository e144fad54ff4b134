"""The C ABI boundary without a GPU: the library loads, exports every symbol the
header declares, and rejects invalid arguments on the host before any launch."""

from __future__ import annotations

import ctypes
import glob
import os
import re

import pytest
import torch

import mla_decode_attention_etap_b200 as m

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names.update(re.findall(r"MLA_API\s+[\w\s\*]*?\b(mla_\w+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_symbols()
    for n in ("mla_decode_plan", "mla_decode_fwd", "mla_combine", "mla_decode_workspace_size"):
        assert n in names


def test_library_exports_every_declared_symbol():
    L = m.lib()
    for n in declared_symbols():
        assert hasattr(L, n), n
    assert set(m.EXPORTS) == set(declared_symbols())


def test_status_strings():
    for code, name in m.STATUS.items():
        assert m.lib().mla_status_string(code).decode() == name


def test_workspace_size_shapes():
    assert m.mla_decode_workspace_size(16, 1, 16, 148) > 0
    big = m.mla_decode_workspace_size(32, 1, 128, 148)
    small = m.mla_decode_workspace_size(32, 1, 16, 148)
    assert big > small
    assert m.lib().mla_decode_workspace_size(0, 1, 16, 148) == 0
    assert m.lib().mla_decode_workspace_size(1, 1, 2048, 148) == 0


# Fake, suitably aligned device addresses: every call below must fail validation
# before touching CUDA, so the pointers are never dereferenced.
A = 1 << 20


def fwd(**kw):
    args = dict(q=A, kv=A, seqlens=A, block_table=None, batch=2, q_len=1, num_heads=16, kv_rows=128,
                max_blocks=0, scale=1 / 24, causal=0, o=A, lse=A, ws=A, ws_bytes=1 << 30, n_sms=148, flags=0)
    args.update(kw)
    vp = ctypes.c_void_p
    return m.lib().mla_decode_fwd(vp(args["q"]), vp(args["kv"]), vp(args["seqlens"]),
                                  vp(args["block_table"]) if args["block_table"] else None, args["batch"],
                                  args["q_len"], args["num_heads"], args["kv_rows"], args["max_blocks"],
                                  ctypes.c_float(args["scale"]), args["causal"], vp(args["o"]), vp(args["lse"]),
                                  vp(args["ws"]), args["ws_bytes"], args["n_sms"], args["flags"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1), (dict(kv=0), -1), (dict(o=0), -1), (dict(lse=0), -1), (dict(ws=0), -1),
    (dict(scale=0.0), -1), (dict(scale=-1.0), -1), (dict(scale=float("inf")), -1), (dict(scale=float("nan")), -1),
    (dict(causal=2), -1), (dict(flags=8), -1), (dict(flags=0x20000000), -1), (dict(batch=0), -1), (dict(q_len=0), -1),
    (dict(num_heads=2048), -2), (dict(kv_rows=0), -1),
    (dict(q=A + 8), -3), (dict(kv=A + 2), -3), (dict(o=A + 4), -3), (dict(lse=A + 2), -3), (dict(ws=A + 16), -3),
    (dict(ws_bytes=100), -4),
    (dict(block_table=A, kv_rows=100, max_blocks=2), -1),      # paged pool not a multiple of 64 rows
    (dict(block_table=A, kv_rows=128, max_blocks=0), -1),
    (dict(block_table=A + 2, kv_rows=128, max_blocks=2), -3),
    (dict(batch=65536, kv_rows=1 << 20), -2),                  # contiguous rows past int32
])
def test_fwd_rejects(kw, code):
    assert fwd(**kw) == code


def test_plan_and_combine_reject():
    L = m.lib()
    vp = ctypes.c_void_p
    assert L.mla_decode_plan(None, 2, 1, 16, 148, vp(A), 1 << 30, None) == -1
    assert L.mla_decode_plan(vp(A), 2, 1, 16, 148, vp(A + 64), 1 << 30, None) == -3
    assert L.mla_decode_plan(vp(A), 2, 1, 16, 148, vp(A), 10, None) == -4
    assert L.mla_combine(None, 2, 1, 16, 148, vp(A), vp(A), None) == -1
    assert L.mla_combine(vp(A), 2, 1, 16, 148, vp(A + 2), vp(A), None) == -3
    out = ctypes.c_int(0)
    assert L.mla_decode_read_status(None, ctypes.byref(out), None) == -1


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(m, "_lib", None)
    monkeypatch.setattr(m, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(ImportError):
        m.lib()


def fwd_fp8(**kw):
    args = dict(q=A, kv8=A, kv_scale=A, seqlens=A, q_lens=None, block_table=None, batch=2, q_len=1, num_heads=16,
                kv_rows=128, max_blocks=0, scale=1 / 24, causal=0, o=A, lse=A, ws=A, ws_bytes=1 << 30, n_sms=148,
                flags=0)
    args.update(kw)
    vp = ctypes.c_void_p
    opt = lambda x: vp(x) if x else None  # noqa: E731
    return m.lib().mla_decode_fwd_fp8(vp(args["q"]), opt(args["kv8"]), opt(args["kv_scale"]), vp(args["seqlens"]),
                                      opt(args["q_lens"]), opt(args["block_table"]), args["batch"], args["q_len"],
                                      args["num_heads"], args["kv_rows"], args["max_blocks"],
                                      ctypes.c_float(args["scale"]), args["causal"], vp(args["o"]), vp(args["lse"]),
                                      vp(args["ws"]), args["ws_bytes"], args["n_sms"], args["flags"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(kv_scale=0), -1),                     # the FP8 entry needs its row scales
    (dict(kv8=0), -1),
    (dict(num_heads=2048), -2),                 # more than MLA_MAX_COLUMNS query columns
    (dict(scale=0.0), -1), (dict(causal=3), -1),
    (dict(kv8=A + 8), -3), (dict(kv_scale=A + 2), -3), (dict(q_lens=A + 2), -3),
    (dict(ws_bytes=100), -4),
])
def test_fwd_fp8_rejects(kw, code):
    assert fwd_fp8(**kw) == code


def test_measurement_helpers_reject():
    L = m.lib()
    vp = ctypes.c_void_p
    ok = dict(form=0, heads=16, streams=3, tiles=8, ctas=2, cycles=A, err=A)

    def abl(**kw):
        a = dict(ok, **kw)
        return L.mla_form_ablation(a["form"], a["heads"], a["streams"], a["tiles"], a["ctas"],
                                   vp(a["cycles"]) if a["cycles"] else None, vp(a["err"]) if a["err"] else None,
                                   None)
    for kw in (dict(form=2), dict(heads=48), dict(streams=0), dict(streams=4), dict(tiles=0), dict(ctas=0),
               dict(cycles=0), dict(err=0)):
        assert abl(**kw) == -1, kw
    assert abl(cycles=A + 4) == -3
    assert abl(err=A + 2) == -3
    assert L.mla_stream_probe(vp(A), 100, 74, vp(A), None) == -1      # rows not a multiple of 128
    assert L.mla_stream_probe(vp(A), 256, 0, vp(A), None) == -1
    assert L.mla_stream_probe(vp(A + 8), 256, 74, vp(A), None) == -3


# ---------------------------------------------------------------------------- binding-level guards
def _decode_args(B=2, q_len=1, h=16, rows=130, paged=False, fp8=False):
    kv_shape = (3, 64, 576) if paged else (B, rows, 576)
    a = dict(q=torch.zeros(B, q_len, h, 576, dtype=torch.bfloat16),
             kv=torch.zeros(kv_shape, dtype=torch.uint8 if fp8 else torch.bfloat16),
             seqlens=torch.zeros(B, dtype=torch.int32),
             block_table=torch.zeros(B, 3, dtype=torch.int32) if paged else None,
             o=torch.zeros(B, q_len, h, 512, dtype=torch.bfloat16),
             lse=torch.zeros(B, q_len, h, dtype=torch.float32),
             workspace=torch.zeros(1024, dtype=torch.uint8),
             q_lens=None,
             kv_scale=torch.ones(kv_shape[:2], dtype=torch.float32) if fp8 else None)
    return a


@pytest.mark.parametrize("paged,fp8", [(False, False), (True, False), (False, True), (True, True)])
def test_decode_guards_accept_well_formed_arguments(paged, fp8):
    m.check_decode_args(**_decode_args(paged=paged, fp8=fp8))


BAD = [
    ("q", lambda a: a["q"].float(), TypeError),
    ("q", lambda a: a["q"][..., :512].contiguous(), ValueError),
    ("q", lambda a: torch.zeros(2, 1, 16, 1152, dtype=torch.bfloat16)[..., ::2], ValueError),  # strided view
    ("kv", lambda a: a["kv"][:1], ValueError),              # fewer cache rows than sequences
    ("kv", lambda a: a["kv"].to(torch.float16), TypeError),
    ("seqlens", lambda a: a["seqlens"].long(), TypeError),
    ("seqlens", lambda a: a["seqlens"][:1], ValueError),
    ("o", lambda a: a["o"][:, :, :, :256].contiguous(), ValueError),
    ("o", lambda a: a["o"].float(), TypeError),
    ("lse", lambda a: a["lse"][:1], ValueError),
    ("q_lens", lambda a: torch.zeros(1, dtype=torch.int32), ValueError),
    ("workspace", lambda a: a["workspace"][::2], ValueError),
]


@pytest.mark.parametrize("name,make,exc", BAD)
def test_decode_guards_reject(name, make, exc):
    a = _decode_args()
    a[name] = make(a)
    with pytest.raises(exc):
        m.check_decode_args(**a)


def test_decode_guards_reject_paged_and_fp8_mistakes():
    a = _decode_args(paged=True)
    a["block_table"] = a["block_table"][:1]
    with pytest.raises(ValueError):
        m.check_decode_args(**a)
    a = _decode_args(fp8=True)
    a["kv_scale"] = a["kv_scale"][:1]
    with pytest.raises(ValueError):
        m.check_decode_args(**a)
    a = _decode_args(fp8=True)
    a["kv"] = a["kv"].to(torch.bfloat16)
    with pytest.raises(TypeError):
        m.check_decode_args(**a)


def test_wrappers_refuse_host_tensors_before_any_launch():
    a = _decode_args()
    with pytest.raises(ValueError, match="CUDA"):
        m.mla_decode_fwd(a["q"], a["kv"], a["seqlens"], None, 0.04, False, a["o"], a["lse"], a["workspace"], 148)
    with pytest.raises(ValueError, match="CUDA"):
        m.mla_decode_plan(a["seqlens"], 1, 16, a["workspace"], 148)
    with pytest.raises(ValueError, match="CUDA"):
        m.mla_combine(a["workspace"], 2, 1, 16, 148, a["o"], a["lse"])


@pytest.mark.parametrize("kw", [dict(), dict(paged=True), dict(kv_dtype="e4m3"), dict(paged=True, kv_dtype="e4m3"),
                                dict(q_len=4, causal=True, q_lens=[4, 1, 3]), dict(num_heads=128, paged=True)])
def test_decode_guards_accept_what_the_parity_tests_pass(kw):
    """The arguments tests/parity.py builds for the GPU (here on the host) pass the binding's guards."""
    from mla_decode_attention_etap_b200 import workloads as W
    kw = dict(kw)
    heads = kw.pop("num_heads", 16)
    w = W.make_workload(3, heads, [700, 5, 130], seed=3, **kw)
    o = torch.full((w.batch, w.q_len, w.num_heads, 512), float("nan"), dtype=torch.bfloat16)
    lse = torch.full((w.batch, w.q_len, w.num_heads), float("nan"), dtype=torch.float32)
    ws = torch.empty(4096, dtype=torch.uint8)
    if w.fp8:
        m.check_decode_args(w.q, w.kv8, w.seqlens, w.block_table, o, lse, ws, w.q_lens, kv_scale=w.kv_scale)
    else:
        m.check_decode_args(w.q, w.kv, w.seqlens, w.block_table, o, lse, ws, w.q_lens)


def test_trace_buffer_layout_and_decoders():
    """The trace buffer holds [2 CTAs][5 roles][cap] event words, then [n_sms][4] span stamps; the
    decoders split them, order events by time and make spans relative to the earliest entry."""
    cap, n_sms = 4, 3
    t = m.trace_buffer(cap, n_sms)
    assert t.dtype == torch.int64 and t.numel() == 2 * 5 * cap + 4 * n_sms and int(t.abs().sum()) == 0
    rows = t[:2 * 5 * cap].view(2, 5, cap)
    word = lambda code, idx, ns: (code << 56) | (idx << 40) | ns
    rows[0, 3, 0] = word(50, 7, 1000)
    rows[0, 3, 1] = word(51, 7, 1900)
    rows[1, 0, 0] = word(57, 0, 1500)
    spans = t[2 * 5 * cap:].view(n_sms, 4)
    spans[0] = torch.tensor([10_000, 10_600, 30_000, 31_000])
    spans[1] = torch.tensor([10_200, 10_700, 29_000, 29_500])
    ev = m.decode_trace_events(t, n_sms)
    assert [(e[0], e[1], e[2], e[3]) for e in ev] == [(0, 3, 50, 7), (1, 0, 57, 0), (0, 3, 51, 7)]
    assert [e[4] for e in ev] == [0, 500, 900]
    sp = m.decode_trace_spans(t, n_sms)
    assert sp[0].tolist() == [0, 600, 20_000, 21_000] and sp[1].tolist() == [200, 700, 19_000, 19_500]
    assert sp[2].tolist() == [0, 0, 0, 0]  # a CTA that did not run stays zero


def test_untransposed_and_trace_entry_points_validate_on_the_host():
    """The two measurement entry points refuse bad arguments before any launch."""
    L = m.lib()
    # null pointers
    rc = L.mla_decode_fwd_untransposed(None, None, None, None, 1, 1, 16, 64, 0, ctypes.c_float(0.1), 0, None, None,
                                       None, 0, 148, 0, None)
    assert rc == -1
    rc = L.mla_decode_fwd_trace(None, None, None, None, 1, 1, 16, 64, 0, ctypes.c_float(0.1), 0, None, None, None,
                                0, 148, None, 16, None)
    assert rc == -1
