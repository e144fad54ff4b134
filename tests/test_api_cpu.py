"""The C ABI boundary without a GPU: the library loads, exports every symbol the
header declares, and rejects invalid arguments on the host before any launch."""

from __future__ import annotations

import ctypes
import glob
import os
import re

import pytest

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
