"""ctypes binding of libtiledattn (argument marshalling only).

Every function here has the name of the C entry point it calls and takes
torch tensors (device memory) or raw integers.  All computation happens in the
CUDA library; there is no Python or CPU fallback -- if the library cannot be
loaded, or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# TILEDATTN_LIB selects another build of the same library (tuning sweeps)
LIB_PATH = os.environ.get("TILEDATTN_LIB") or os.path.join(_PKG, "libtiledattn.so")

ATTN_OK = 0
STATUS_NAMES = {0: "ATTN_OK", -1: "ATTN_ERR_INVALID_ARG", -2: "ATTN_ERR_UNSUPPORTED",
                -3: "ATTN_ERR_MISALIGNED", -4: "ATTN_ERR_CUDA", -5: "ATTN_ERR_TIMEOUT",
                -6: "ATTN_ERR_TOO_LARGE", -7: "ATTN_ERR_BOUNDS"}

# (name, restype, argtypes)
_VP, _I, _F, _SZ, _ULL = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_ulonglong
SIGNATURES = [
    ("attn_status_string", ctypes.c_char_p, [_I]),
    ("attn_version", ctypes.c_char_p, []),
    ("attn_fwd", _I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _VP]),
    ("attn_decode_workspace_bytes", _SZ, [_I, _I, _I, _I]),
    ("attn_decode", _I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _VP, _SZ, _VP]),
    ("attn_decode_noalloc", _I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _VP]),
    ("attn_fwd_gqa", _I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _F, _VP]),
    ("attn_bwd_workspace_bytes", _SZ, [_I, _I, _I]),
    ("attn_bwd", _I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _VP, _SZ, _VP]),
    ("attn_bwd_fp8p", _I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _VP, _SZ, _VP]),
    ("attn_decode_gqa", _I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _VP, _SZ, _VP]),
    ("attn_fwd_varlen", _I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _I, _F, _VP]),
    ("attn_decode_varlen", _I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _VP, _SZ, _VP]),
    ("attn_quantize_int8", _I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _VP]),
    ("attn_quantize_int4", _I, [_VP, _VP, _VP, _I, _I, _I, _I, _VP]),
    ("attn_fwd_int8", _I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _VP]),
    ("attn_int8_scores", _I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _VP]),
    ("attn_nvfp4_codes_bytes", _SZ, [_I, _I, _I, _I, _I]),
    ("attn_nvfp4_sf_bytes", _SZ, [_I, _I, _I, _I, _I]),
    ("attn_quantize_nvfp4", _I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _VP]),
    ("attn_fwd_fp4", _I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _I, _VP]),
    ("attn_fp4_scores", _I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _VP]),
    ("attn_quantize_fp8", _I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _VP, _VP]),
    ("attn_fwd_fp8", _I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _I, _VP]),
    ("attn_check_status", _I, [_VP]),
    ("attn_set_wait_limit_ns", None, [_ULL]),
    ("attn_watchdog_selftest", _I, [_ULL, _VP]),
    ("attn_debug_counters", _I, [_VP, _I]),
]

_lib = None


class AttnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)}")
        self.code = code


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the shared library (once) and declare every entry point."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing; build it with `python -m tiled_attention_24_b200.build`")
    lib = ctypes.CDLL(path)
    for name, res, args in SIGNATURES:
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(fn, rc):
    if rc != ATTN_OK:
        raise AttnError(fn, rc)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


_BF16, _F32, _I8, _U8, _I32 = torch.bfloat16, torch.float32, torch.int8, torch.uint8, torch.int32


def _expect(*specs):
    """(tensor, shape, dtype, name) tuples: every buffer must have exactly the
    shape and dtype the call implies, so that no kernel writes or reads past a
    caller's tensor (the C ABI sees only pointers and the sizes passed here)."""
    for t, shape, dtype, name in specs:
        if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
            raise ValueError(f"{name}: expected {tuple(shape)} {dtype}, got {tuple(t.shape)} {t.dtype}")


def _at_least(t, nbytes: int, name: str):
    if t.numel() * t.element_size() < nbytes:
        raise ValueError(f"{name}: needs {nbytes} bytes, got {t.numel() * t.element_size()}")


def attn_fwd(q, k, v, o, lse, causal: bool, scale: float, stream=None):
    """bf16 forward: q [B,H,Nq,d], k/v [B,H,Nkv,d] -> o (bf16), lse (fp32)."""
    _need_cuda(q, k, v, o, lse)
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    _expect((q, (B, H, Nq, d), _BF16, "q"), (k, (B, H, Nkv, d), _BF16, "k"), (v, (B, H, Nkv, d), _BF16, "v"),
            (o, (B, H, Nq, d), _BF16, "o"), (lse, (B, H, Nq), _F32, "lse"))
    rc = load().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nkv, d, int(bool(causal)),
                         float(scale), _stream(stream))
    _check("attn_fwd", rc)


def attn_fwd_gqa(q, k, v, o, lse, causal: bool, scale: float, stream=None):
    """Grouped-query forward: q [B,Hq,Nq,d], k/v [B,Hkv,Nkv,d] (Hq % Hkv == 0)."""
    _need_cuda(q, k, v, o, lse)
    B, Hq, Nq, d = q.shape
    Hkv, Nkv = k.shape[1], k.shape[2]
    _expect((q, (B, Hq, Nq, d), _BF16, "q"), (k, (B, Hkv, Nkv, d), _BF16, "k"), (v, (B, Hkv, Nkv, d), _BF16, "v"),
            (o, (B, Hq, Nq, d), _BF16, "o"), (lse, (B, Hq, Nq), _F32, "lse"))
    rc = load().attn_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nkv, d,
                             int(bool(causal)), float(scale), _stream(stream))
    _check("attn_fwd_gqa", rc)


def attn_decode_gqa(q, k, v, o, lse, scale: float, num_splits: int, workspace, stream=None):
    """Grouped-query split-KV decode: q [B,Hq,1,d], k/v [B,Hkv,Nkv,d]."""
    _need_cuda(q, k, v, o, lse, workspace)
    B, Hq, _, d = q.shape
    Hkv, Nkv = k.shape[1], k.shape[2]
    _expect((q, (B, Hq, 1, d), _BF16, "q"), (k, (B, Hkv, Nkv, d), _BF16, "k"), (v, (B, Hkv, Nkv, d), _BF16, "v"),
            (o, (B, Hq, 1, d), _BF16, "o"), (lse, (B, Hq, 1), _F32, "lse"))
    rc = load().attn_decode_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nkv, d, float(scale),
                                int(num_splits), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream))
    _check("attn_decode_gqa", rc)


def attn_bwd_workspace_bytes(B: int, H: int, Nq: int) -> int:
    return int(load().attn_bwd_workspace_bytes(B, H, Nq))


def attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, causal: bool, scale: float, workspace, stream=None):
    """bf16 backward: gradients dq, dk, dv of the forward (o, lse) for upstream dout."""
    _need_cuda(q, k, v, o, dout, lse, dq, dk, dv, workspace)
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    _expect((q, (B, H, Nq, d), _BF16, "q"), (k, (B, H, Nkv, d), _BF16, "k"), (v, (B, H, Nkv, d), _BF16, "v"),
            (o, (B, H, Nq, d), _BF16, "o"), (dout, (B, H, Nq, d), _BF16, "dout"), (lse, (B, H, Nq), _F32, "lse"),
            (dq, (B, H, Nq, d), _BF16, "dq"), (dk, (B, H, Nkv, d), _BF16, "dk"), (dv, (B, H, Nkv, d), _BF16, "dv"))
    rc = load().attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                         B, H, Nq, Nkv, d, int(bool(causal)), float(scale), _ptr(workspace),
                         workspace.numel() * workspace.element_size(), _stream(stream))
    _check("attn_bwd", rc)


def attn_bwd_fp8p(q, k, v, o, dout, lse, dq, dk, dv, causal: bool, scale: float, workspace, stream=None):
    """attn_bwd with P rounded to e4m3 before dV = P^T dO (the FP8-P backward)."""
    _need_cuda(q, k, v, o, dout, lse, dq, dk, dv, workspace)
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    _expect((q, (B, H, Nq, d), _BF16, "q"), (k, (B, H, Nkv, d), _BF16, "k"), (v, (B, H, Nkv, d), _BF16, "v"),
            (o, (B, H, Nq, d), _BF16, "o"), (dout, (B, H, Nq, d), _BF16, "dout"), (lse, (B, H, Nq), _F32, "lse"),
            (dq, (B, H, Nq, d), _BF16, "dq"), (dk, (B, H, Nkv, d), _BF16, "dk"), (dv, (B, H, Nkv, d), _BF16, "dv"))
    rc = load().attn_bwd_fp8p(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                              _ptr(dv), B, H, Nq, Nkv, d, int(bool(causal)), float(scale), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    _check("attn_bwd_fp8p", rc)


def attn_decode_workspace_bytes(B: int, H: int, d: int, num_splits: int) -> int:
    return int(load().attn_decode_workspace_bytes(B, H, d, num_splits))


def attn_decode(q, k, v, o, lse, scale: float, num_splits: int, workspace, stream=None):
    """Split-KV decode: q [B,H,1,d], k/v [B,H,Nkv,d] -> o [B,H,1,d], lse [B,H,1]."""
    _need_cuda(q, k, v, o, lse, workspace)
    B, H, _, d = q.shape
    Nkv = k.shape[2]
    _expect((q, (B, H, 1, d), _BF16, "q"), (k, (B, H, Nkv, d), _BF16, "k"), (v, (B, H, Nkv, d), _BF16, "v"),
            (o, (B, H, 1, d), _BF16, "o"), (lse, (B, H, 1), _F32, "lse"))
    rc = load().attn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nkv, d, float(scale),
                            int(num_splits), _ptr(workspace), workspace.numel() * workspace.element_size(),
                            _stream(stream))
    _check("attn_decode", rc)


def attn_decode_noalloc(q, k, v, o, lse, scale: float, num_splits: int, stream=None):
    """attn_decode with the library's fixed scratch instead of a workspace
    (for callers that cannot allocate device memory)."""
    _need_cuda(q, k, v, o, lse)
    B, H, _, d = q.shape
    Nkv = k.shape[2]
    _expect((q, (B, H, 1, d), _BF16, "q"), (k, (B, H, Nkv, d), _BF16, "k"), (v, (B, H, Nkv, d), _BF16, "v"),
            (o, (B, H, 1, d), _BF16, "o"), (lse, (B, H, 1), _F32, "lse"))
    rc = load().attn_decode_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nkv, d, float(scale),
                                    int(num_splits), _stream(stream))
    _check("attn_decode_noalloc", rc)


def attn_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, max_seqlen_q: int, causal: bool, scale: float, stream=None):
    """Packed variable-length forward: q/o [total_q,H,d], k/v [total_k,Hkv,d] bf16,
    lse [H,total_q] fp32, cu_q/cu_k int32 [B+1] on the device."""
    _need_cuda(q, k, v, o, lse, cu_q, cu_k)
    total_q, H, d = q.shape
    total_k, Hkv, _ = k.shape
    B = cu_q.shape[0] - 1
    _expect((q, (total_q, H, d), _BF16, "q"), (k, (total_k, Hkv, d), _BF16, "k"), (v, (total_k, Hkv, d), _BF16, "v"),
            (o, (total_q, H, d), _BF16, "o"), (lse, (H, total_q), _F32, "lse"), (cu_q, (B + 1,), _I32, "cu_q"),
            (cu_k, (B + 1,), _I32, "cu_k"))
    rc = load().attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_q), _ptr(cu_k), B, H, Hkv,
                                total_q, total_k, int(max_seqlen_q), d, int(bool(causal)), float(scale),
                                _stream(stream))
    _check("attn_fwd_varlen", rc)


def attn_decode_varlen(q, k, v, o, lse, seqlens_k, scale: float, num_splits: int, workspace, stream=None):
    """Decode with a cache length per batch entry: q [B,H,1,d], k/v [B,Hkv,Nkv_max,d],
    seqlens_k int32 [B] on the device."""
    _need_cuda(q, k, v, o, lse, seqlens_k, workspace)
    B, H, _, d = q.shape
    Hkv, Nkv = k.shape[1], k.shape[2]
    _expect((q, (B, H, 1, d), _BF16, "q"), (k, (B, Hkv, Nkv, d), _BF16, "k"), (v, (B, Hkv, Nkv, d), _BF16, "v"),
            (o, (B, H, 1, d), _BF16, "o"), (lse, (B, H, 1), _F32, "lse"), (seqlens_k, (B,), _I32, "seqlens_k"))
    rc = load().attn_decode_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(seqlens_k), B, H, Hkv, Nkv,
                                   d, float(scale), int(num_splits), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check("attn_decode_varlen", rc)


def attn_quantize_int8(x, xq, xs, per_head: bool, stream=None):
    """bf16 [B,H,N,d] -> int8 xq, fp32 xs ([B,H,N] per token or [B,H] per head)."""
    _need_cuda(x, xq, xs)
    B, H, N, d = x.shape
    _expect((x, (B, H, N, d), _BF16, "x"), (xq, (B, H, N, d), _I8, "xq"),
            (xs, (B, H) if per_head else (B, H, N), _F32, "xs"))
    _check("attn_quantize_int8", load().attn_quantize_int8(_ptr(x), _ptr(xq), _ptr(xs), B, H, N, d,
                                                             int(bool(per_head)), _stream(stream)))


def attn_quantize_int4(x, xq, xs, stream=None):
    """bf16 [B,H,N,d] -> INT4 codes in int8 containers, fp32 per-token scales."""
    _need_cuda(x, xq, xs)
    B, H, N, d = x.shape
    _expect((x, (B, H, N, d), _BF16, "x"), (xq, (B, H, N, d), _I8, "xq"), (xs, (B, H, N), _F32, "xs"))
    _check("attn_quantize_int4", load().attn_quantize_int4(_ptr(x), _ptr(xq), _ptr(xs), B, H, N, d, _stream(stream)))


def attn_fwd_int8(q, qs, k, ks, v, vs, o, lse, causal: bool, scale: float, stream=None):
    """INT8 forward: int8 q/k/v [B,H,N,128] with scales -> o fp32, lse fp32."""
    _need_cuda(q, qs, k, ks, v, vs, o, lse)
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    _expect((q, (B, H, Nq, d), _I8, "q"), (k, (B, H, Nkv, d), _I8, "k"), (v, (B, H, Nkv, d), _I8, "v"),
            (qs, (B, H, Nq), _F32, "q_scale"), (ks, (B, H, Nkv), _F32, "k_scale"), (vs, (B, H), _F32, "v_scale"),
            (o, (B, H, Nq, d), _F32, "o"), (lse, (B, H, Nq), _F32, "lse"))
    rc = load().attn_fwd_int8(_ptr(q), _ptr(qs), _ptr(k), _ptr(ks), _ptr(v), _ptr(vs), _ptr(o), _ptr(lse),
                              B, H, Nq, Nkv, d, int(bool(causal)), float(scale), _stream(stream))
    _check("attn_fwd_int8", rc)


def attn_int8_scores(q, k, s, stream=None):
    """int32 S = q k^T of int8 [B,H,N,128] operands, through the INT8 MMA path."""
    _need_cuda(q, k, s)
    B, H, Nq, d = q.shape
    _expect((q, (B, H, Nq, d), _I8, "q"), (k, (B, H, k.shape[2], d), _I8, "k"),
            (s, (B, H, Nq, k.shape[2]), _I32, "s"))
    _check("attn_int8_scores", load().attn_int8_scores(_ptr(q), _ptr(k), _ptr(s), B, H, Nq, k.shape[2], d,
                                                         _stream(stream)))


def attn_nvfp4_codes_bytes(B: int, H: int, N: int, d: int, mode: int) -> int:
    return int(load().attn_nvfp4_codes_bytes(B, H, N, d, mode))


def attn_nvfp4_sf_bytes(B: int, H: int, N: int, d: int, mode: int) -> int:
    return int(load().attn_nvfp4_sf_bytes(B, H, N, d, mode))


def attn_quantize_nvfp4(x, codes, sf, mode: int, stream=None):
    """bf16 [B,H,N,128] -> packed e2m1 codes + tiled e4m3 scales (mode 0: Q/K, 1: V^T)."""
    _need_cuda(x, codes, sf)
    B, H, N, d = x.shape
    _expect((x, (B, H, N, d), _BF16, "x"))
    _at_least(codes, attn_nvfp4_codes_bytes(B, H, N, d, mode), "codes")
    _at_least(sf, attn_nvfp4_sf_bytes(B, H, N, d, mode), "sf")
    _check("attn_quantize_nvfp4", load().attn_quantize_nvfp4(_ptr(x), _ptr(codes), _ptr(sf), B, H, N, d, int(mode),
                                                               _stream(stream)))


def attn_fwd_fp4(q, qsf, k, ksf, vt, vtsf, o, lse, B, H, Nq, Nkv, causal: bool, scale: float, p_mode: int,
                 stream=None):
    """FP4 forward (codes/scales from attn_quantize_nvfp4) -> o fp32 [B,H,Nq,128], lse fp32."""
    _need_cuda(q, qsf, k, ksf, vt, vtsf, o, lse)
    for t, n, m, nm in ((q, Nq, 0, "q"), (k, Nkv, 0, "k"), (vt, Nkv, 1, "vt")):
        _at_least(t, attn_nvfp4_codes_bytes(B, H, n, 128, m), nm)
    for t, n, m, nm in ((qsf, Nq, 0, "q_sf"), (ksf, Nkv, 0, "k_sf"), (vtsf, Nkv, 1, "vt_sf")):
        _at_least(t, attn_nvfp4_sf_bytes(B, H, n, 128, m), nm)
    _expect((o, (B, H, Nq, 128), _F32, "o"), (lse, (B, H, Nq), _F32, "lse"))
    rc = load().attn_fwd_fp4(_ptr(q), _ptr(qsf), _ptr(k), _ptr(ksf), _ptr(vt), _ptr(vtsf), _ptr(o), _ptr(lse),
                             B, H, Nq, Nkv, 128, int(bool(causal)), float(scale), int(p_mode), _stream(stream))
    _check("attn_fwd_fp4", rc)


def attn_fp4_scores(q, qsf, k, ksf, s, B, H, Nq, Nkv, stream=None):
    """fp32 S = deq(q) deq(k)^T through the block-scaled FP4 MMA path."""
    _need_cuda(q, qsf, k, ksf, s)
    for t, n, nm in ((q, Nq, "q"), (k, Nkv, "k")):
        _at_least(t, attn_nvfp4_codes_bytes(B, H, n, 128, 0), nm)
    for t, n, nm in ((qsf, Nq, "q_sf"), (ksf, Nkv, "k_sf")):
        _at_least(t, attn_nvfp4_sf_bytes(B, H, n, 128, 0), nm)
    _expect((s, (B, H, Nq, Nkv), _F32, "s"))
    _check("attn_fp4_scores", load().attn_fp4_scores(_ptr(q), _ptr(qsf), _ptr(k), _ptr(ksf), _ptr(s), B, H, Nq, Nkv,
                                                       128, _stream(stream)))


def attn_quantize_fp8(x, codes, scales, mode: int, signs=None, stream=None):
    """bf16 [B,H,N,d] -> e4m3 codes (uint8) + fp32 scales; mode 0: per row
    ([B,H,N]; rotated by H_d diag(signs) when signs is given), 1: per channel ([B,H,d])."""
    _need_cuda(x, codes, scales)
    if signs is not None:
        _need_cuda(signs)
    B, H, N, d = x.shape
    _expect((x, (B, H, N, d), _BF16, "x"), (codes, (B, H, N, d), _U8, "codes"),
            (scales, (B, H, N) if mode == 0 else (B, H, d), _F32, "scales"))
    if signs is not None:
        _expect((signs, (d,), _F32, "signs"))
    _check("attn_quantize_fp8", load().attn_quantize_fp8(_ptr(x), _ptr(codes), _ptr(scales), B, H, N, d, int(mode),
                                                           None if signs is None else _ptr(signs),
                                                           _stream(stream)))


def attn_fwd_fp8(q, qs, k, ks, v, vs, o, lse, causal: bool, scale: float, rotated: bool, stream=None):
    """FP8 forward: e4m3 codes [B,H,N,128] with scales -> o fp32, lse fp32."""
    _need_cuda(q, qs, k, ks, v, vs, o, lse)
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    _expect((q, (B, H, Nq, d), _U8, "q"), (k, (B, H, Nkv, d), _U8, "k"), (v, (B, H, Nkv, d), _U8, "v"),
            (qs, (B, H, Nq), _F32, "q_scale"), (ks, (B, H, Nkv), _F32, "k_scale"), (vs, (B, H, d), _F32, "v_scale"),
            (o, (B, H, Nq, d), _F32, "o"), (lse, (B, H, Nq), _F32, "lse"))
    rc = load().attn_fwd_fp8(_ptr(q), _ptr(qs), _ptr(k), _ptr(ks), _ptr(v), _ptr(vs), _ptr(o), _ptr(lse),
                             B, H, Nq, Nkv, d, int(bool(causal)), float(scale), int(bool(rotated)),
                             _stream(stream))
    _check("attn_fwd_fp8", rc)


def attn_check_status(stream=None) -> int:
    return int(load().attn_check_status(_stream(stream)))


def attn_set_wait_limit_ns(ns: int) -> None:
    load().attn_set_wait_limit_ns(int(ns))


def attn_watchdog_selftest(limit_ns: int, stream=None) -> None:
    _check("attn_watchdog_selftest", load().attn_watchdog_selftest(int(limit_ns), _stream(stream)))


def attn_debug_counters(reset: bool = False):
    """The debug build's four counters (rescales, skipped causal tiles, bounds
    violations, reserved); raises AttnError(ATTN_ERR_UNSUPPORTED) in the
    product build."""
    buf = (ctypes.c_ulonglong * 4)()
    _check("attn_debug_counters", load().attn_debug_counters(ctypes.cast(buf, _VP), int(bool(reset))))
    return [int(x) for x in buf]


def attn_version() -> str:
    return load().attn_version().decode()


def attn_status_string(code: int) -> str:
    return load().attn_status_string(int(code)).decode()
