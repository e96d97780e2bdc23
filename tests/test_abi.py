"""The C-ABI library loads without a GPU, exports every entry point that
include/tiledattn.h declares, and rejects bad arguments on the host before
touching the device.  No GPU (no call here reaches CUDA)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(attn_\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    from tiled_attention_24_b200 import build
    build.build()
    from tiled_attention_24_b200 import _binding
    return _binding.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"attn_fwd", "attn_decode", "attn_check_status"} <= names
    for n in sorted(names):
        assert hasattr(lib, n), n


def test_binding_covers_every_declared_symbol():
    from tiled_attention_24_b200 import _binding
    assert _declared() == {n for n, _, _ in _binding.SIGNATURES}


def test_status_strings(lib):
    assert lib.attn_status_string(0) == b"ATTN_OK"
    assert lib.attn_status_string(-5) == b"ATTN_ERR_TIMEOUT"
    assert b"sm_100a" in lib.attn_version()


P = ctypes.c_void_p(16 * 1000)  # never dereferenced: validation rejects first


@pytest.mark.parametrize("args,code", [
    (dict(d=96), -2), (dict(d=32), -2), (dict(scale=0.0), -1), (dict(scale=float("nan")), -1),
    (dict(scale=-1.0), -1), (dict(B=-1), -1), (dict(Nq=-3), -1), (dict(q=None), -1),
    (dict(q=ctypes.c_void_p(16 * 1000 + 2)), -3), (dict(lse=ctypes.c_void_p(16 * 1000 + 1)), -3),
    (dict(B=0), 0), (dict(Nq=0), 0),
])
def test_fwd_host_validation(lib, args, code):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=1, Nq=8, Nkv=8, d=64, causal=0, scale=0.125, stream=None)
    a.update(args)
    rc = lib.attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Nq"], a["Nkv"],
                      a["d"], a["causal"], a["scale"], a["stream"])
    assert rc == code


def test_decode_workspace_size_and_validation(lib):
    n = lib.attn_decode_workspace_bytes(64, 32, 128, 16)
    assert n >= 64 * 32 * 16 * (128 + 1) * 4
    assert lib.attn_decode_workspace_bytes(1, 1, 96, 4) == 0
    ws = ctypes.c_void_p(16 * 4096)
    def call(**kw):
        a = dict(B=2, H=2, Nkv=100, d=128, scale=0.1, S=4, ws_bytes=n)
        a.update(kw)
        return lib.attn_decode(P, P, P, P, P, a["B"], a["H"], a["Nkv"], a["d"], a["scale"], a["S"], ws,
                               a["ws_bytes"], None)
    assert call(S=0) == -1 and call(S=2000) == -1 and call(Nkv=0) == -1
    assert call(d=80) == -2 and call(ws_bytes=16) == -1 and call(scale=0.0) == -1
    assert call(B=0) == 0


@pytest.mark.parametrize("Hq,Hkv,code", [(8, 3, -1), (8, 0, -1), (4, 8, -1), (8, 2, None), (8, 8, None), (8, 1, None)])
def test_gqa_head_validation(lib, Hq, Hkv, code):
    """Uneven head groups are rejected before anything touches the device;
    valid groups pass validation (checked with d = 96, which then fails as
    unsupported, so nothing is launched)."""
    rc = lib.attn_fwd_gqa(P, P, P, P, P, 1, Hq, Hkv, 8, 8, 64 if code else 96, 0, 0.125, None)
    assert rc == (code if code else -2)
    n = lib.attn_decode_workspace_bytes(1, Hq, 128, 4)
    rc = lib.attn_decode_gqa(P, P, P, P, P, 1, Hq, Hkv, 100, 128 if code else 96, 0.1, 4,
                             ctypes.c_void_p(16 * 4096), n, None)
    assert rc == (code if code else -2)


def test_bwd_workspace_and_validation(lib):
    n = lib.attn_bwd_workspace_bytes(2, 3, 100)
    assert n >= 2 * 3 * 100 * 4 and n % 256 == 0
    assert lib.attn_bwd_workspace_bytes(0, 3, 100) == 0
    ws = ctypes.c_void_p(16 * 4096)
    def call(**kw):
        a = dict(B=1, H=2, Nq=64, Nkv=64, d=128, causal=0, scale=0.1, ws_bytes=n)
        a.update(kw)
        return lib.attn_bwd(P, P, P, P, P, P, P, P, P, a["B"], a["H"], a["Nq"], a["Nkv"], a["d"], a["causal"],
                            a["scale"], ws, a["ws_bytes"], None)
    assert call(d=96) == -2 and call(scale=0.0) == -1 and call(B=-1) == -1 and call(Nkv=-2) == -1
    assert call(ws_bytes=16) == -1 and call(B=0) == 0
    # the FP8-P entry point validates exactly like attn_bwd
    def call8(**kw):
        a = dict(B=1, H=2, Nq=64, Nkv=64, d=128, causal=0, scale=0.1, ws_bytes=n)
        a.update(kw)
        return lib.attn_bwd_fp8p(P, P, P, P, P, P, P, P, P, a["B"], a["H"], a["Nq"], a["Nkv"], a["d"], a["causal"],
                                 a["scale"], ws, a["ws_bytes"], None)
    assert call8(d=96) == -2 and call8(scale=0.0) == -1 and call8(B=-1) == -1 and call8(ws_bytes=16) == -1
    assert call8(B=0) == 0


def test_fp8_host_validation(lib):
    def quant(**kw):
        a = dict(B=1, H=2, N=64, d=128, mode=0, signs=None)
        a.update(kw)
        return lib.attn_quantize_fp8(P, P, P, a["B"], a["H"], a["N"], a["d"], a["mode"], a["signs"], None)
    assert quant(d=96) == -2 and quant(mode=2) == -1 and quant(N=-1) == -1
    assert quant(mode=1, signs=P) == -1 and quant(signs=ctypes.c_void_p(16 * 1000 + 2)) == -3
    assert quant(B=0) == 0
    def fwd(**kw):
        a = dict(B=1, H=2, Nq=64, Nkv=64, d=128, causal=0, scale=0.1, rot=1, vs=P)
        a.update(kw)
        return lib.attn_fwd_fp8(P, P, P, P, P, a["vs"], P, P, a["B"], a["H"], a["Nq"], a["Nkv"], a["d"],
                                a["causal"], a["scale"], a["rot"], None)
    assert fwd(d=64) == -2 and fwd(scale=0.0) == -1 and fwd(Nkv=0) == -2 and fwd(Nq=-1) == -1
    assert fwd(vs=ctypes.c_void_p(16 * 1000 + 4)) == -3 and fwd(Nq=0) == 0


def test_varlen_host_validation(lib):
    def fwd(**kw):
        a = dict(cuq=P, cuk=P, B=2, H=4, Hkv=2, tq=100, tk=100, mq=64, d=128, scale=0.1, q=P)
        a.update(kw)
        return lib.attn_fwd_varlen(a["q"], P, P, P, P, a["cuq"], a["cuk"], a["B"], a["H"], a["Hkv"], a["tq"],
                                   a["tk"], a["mq"], a["d"], 0, a["scale"], None)
    assert fwd(d=96) == -2 and fwd(Hkv=3) == -1 and fwd(cuq=None) == -1 and fwd(tq=-1) == -1
    assert fwd(scale=0.0) == -1 and fwd(q=ctypes.c_void_p(16 * 1000 + 8)) == -3
    assert fwd(cuk=ctypes.c_void_p(16 * 1000 + 2)) == -3 and fwd(tq=0) == 0 and fwd(B=0) == 0
    n = lib.attn_decode_workspace_bytes(2, 4, 128, 4)
    def dec(**kw):
        a = dict(lens=P, B=2, H=4, Hkv=2, N=100, d=128, S=4)
        a.update(kw)
        return lib.attn_decode_varlen(P, P, P, P, P, a["lens"], a["B"], a["H"], a["Hkv"], a["N"], a["d"], 0.1,
                                      a["S"], ctypes.c_void_p(16 * 4096), n, None)
    assert dec(lens=None) == -1 and dec(lens=ctypes.c_void_p(16 * 1000 + 2)) == -3 and dec(d=80) == -2
    assert dec(S=0) == -1 and dec(N=0) == -1 and dec(B=0) == 0


def test_product_path_never_imports_the_oracle():
    """The package must not reach the oracle (no CPU fallback)."""
    pkg = os.path.join(ROOT, "tiled_attention_24_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in src.replace("oracle/", ""), f


def test_debug_counters_only_in_debug_build(lib):
    """The product library answers ATTN_ERR_UNSUPPORTED (before any CUDA
    call); the debug build exports the same entry points and rejects a null
    output on the host."""
    buf = (ctypes.c_ulonglong * 4)()
    assert lib.attn_debug_counters(ctypes.cast(buf, ctypes.c_void_p), 0) == -2
    assert lib.attn_status_string(-7) == b"ATTN_ERR_BOUNDS"
    from tiled_attention_24_b200 import build
    path = build.build_debug()
    dbg = ctypes.CDLL(path)
    for n in sorted(_declared()):
        assert hasattr(dbg, n), n
    dbg.attn_debug_counters.argtypes = [ctypes.c_void_p, ctypes.c_int]
    assert dbg.attn_debug_counters(None, 0) == -1
