"""Fused tiled attention forward for NVIDIA B200 (sm_100a).

The compute lives in ``libtiledattn.so`` (CUDA kernels behind a C ABI, see
``include/tiledattn.h``); this package is its thin ctypes binding plus a few
conveniences that allocate outputs with torch and call the same entry points.
"""
from __future__ import annotations

import math

import torch

from ._binding import (AttnError, LIB_PATH, attn_check_status, attn_debug_counters, attn_decode,  # noqa: F401
                       attn_decode_gqa, attn_decode_noalloc, attn_decode_workspace_bytes, attn_fp4_scores,
                       attn_fwd, attn_fwd_fp8, attn_fwd_gqa, attn_fwd_varlen, attn_decode_varlen, attn_quantize_fp8, attn_quantize_int4, attn_bwd, attn_bwd_fp8p, attn_bwd_workspace_bytes,
                       attn_fwd_fp4, attn_fwd_int8, attn_int8_scores, attn_nvfp4_codes_bytes,
                       attn_nvfp4_sf_bytes, attn_quantize_int8, attn_quantize_nvfp4, attn_set_wait_limit_ns,
                       attn_status_string, attn_version, attn_watchdog_selftest, load)

__all__ = ["load", "attn_fwd", "attn_decode", "attn_decode_workspace_bytes", "attn_check_status",
           "attn_set_wait_limit_ns", "attn_watchdog_selftest", "attn_version", "attn_status_string",
           "AttnError", "forward", "decode", "quantize_int8", "forward_int8",
           "attn_quantize_int8", "attn_fwd_int8", "attn_int8_scores", "attn_decode_noalloc",
           "attn_quantize_nvfp4", "attn_fwd_fp4", "attn_fp4_scores", "quantize_nvfp4", "forward_fp4",
           "attn_fwd_gqa", "attn_decode_gqa", "attn_quantize_int4", "quantize_int4", "forward_int4",
           "attn_bwd", "attn_bwd_fp8p", "attn_bwd_workspace_bytes", "backward",
           "attn_quantize_fp8", "attn_fwd_fp8", "quantize_fp8", "forward_fp8", "hadamard_signs",
           "attn_fwd_varlen", "attn_decode_varlen", "forward_varlen", "decode_varlen",
           "attn_debug_counters", "DIRECT_P", "QUANT_AFTER_EXP"]

DIRECT_P, QUANT_AFTER_EXP = 0, 1


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
            scale: float | None = None, stream=None):
    """Allocate O (bf16) and LSE (fp32) and run ``attn_fwd`` (``attn_fwd_gqa``
    when k/v have fewer heads than q: grouped-query attention)."""
    B, H, Nq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    if k.shape[1] != H:
        attn_fwd_gqa(q, k, v, o, lse, causal, scale, stream)
    else:
        attn_fwd(q, k, v, o, lse, causal, scale, stream)
    return o, lse


def backward(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None, stream=None,
             p_fp8: bool = False):
    """Allocate dq, dk, dv (bf16) and the row-statistic workspace, run ``attn_bwd``
    (``attn_bwd_fp8p`` with ``p_fp8``: P in e4m3 for dV) (o, lse: the
    forward's outputs for the same arguments)."""
    B, H, Nq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(16, attn_bwd_workspace_bytes(B, H, Nq)), dtype=torch.uint8, device=q.device)
    (attn_bwd_fp8p if p_fp8 else attn_bwd)(q, k, v, o, dout, lse, dq, dk, dv, causal, scale, ws, stream)
    return dq, dk, dv


def decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
           num_splits: int = 16, workspace: torch.Tensor | None = None, stream=None):
    """Allocate O, LSE (and a workspace if none is given) and run ``attn_decode``
    (``attn_decode_gqa`` when k/v have fewer heads than q)."""
    B, H, _, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if workspace is None:
        nbytes = attn_decode_workspace_bytes(B, H, d, num_splits)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, 1), dtype=torch.float32, device=q.device)
    if k.shape[1] != H:
        attn_decode_gqa(q, k, v, o, lse, scale, num_splits, workspace, stream)
    else:
        attn_decode(q, k, v, o, lse, scale, num_splits, workspace, stream)
    return o, lse


def forward_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, causal: bool = False,
                   scale: float | None = None, stream=None):
    """Packed variable-length forward (q [total_q,H,d], k/v [total_k,Hkv,d],
    cu_seqlens int32 [B+1] on the device).  Returns (o [total_q,H,d], lse [H,total_q])."""
    total_q, H, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.zeros_like(q)
    lse = torch.full((H, total_q), float("-inf"), dtype=torch.float32, device=q.device)
    attn_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, causal, scale, stream)
    return o, lse


def decode_varlen(q, k, v, seqlens_k, scale: float | None = None, num_splits: int = 16, stream=None):
    """Decode with a cache length per batch entry (seqlens_k int32 [B] on the device)."""
    B, H, _, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    ws = torch.empty(attn_decode_workspace_bytes(B, H, d, num_splits), dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, 1), dtype=torch.float32, device=q.device)
    attn_decode_varlen(q, k, v, o, lse, seqlens_k, scale, num_splits, ws, stream)
    return o, lse


def quantize_int8(x: torch.Tensor, per_head: bool = False, stream=None):
    """INT8 symmetric quantisation (per token row, or per (batch, head))."""
    B, H, N, d = x.shape
    xq = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    xs = torch.empty((B, H) if per_head else (B, H, N), dtype=torch.float32, device=x.device)
    attn_quantize_int8(x, xq, xs, per_head, stream)
    return xq, xs


def forward_int8(q, k, v, causal: bool = False, scale: float | None = None, stream=None):
    """Quantise bf16 q, k (per token) and v (per head) and run the INT8 forward.
    Returns (o fp32, lse fp32)."""
    B, H, Nq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    qi, qs = quantize_int8(q, False, stream)
    ki, ks = quantize_int8(k, False, stream)
    vi, vs = quantize_int8(v, True, stream)
    o = torch.empty((B, H, Nq, d), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    attn_fwd_int8(qi, qs, ki, ks, vi, vs, o, lse, causal, scale, stream)
    return o, lse


def quantize_int4(x: torch.Tensor, stream=None):
    """Token-level INT4 quantisation (codes in [-7, 7], int8 containers)."""
    B, H, N, d = x.shape
    xq = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    xs = torch.empty((B, H, N), dtype=torch.float32, device=x.device)
    attn_quantize_int4(x, xq, xs, stream)
    return xq, xs


def forward_int4(q, k, v, causal: bool = False, scale: float | None = None, stream=None):
    """INT4 q, k (per token), INT8 v (per head), through the INT8 forward.
    Returns (o fp32, lse fp32)."""
    B, H, Nq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    qi, qs = quantize_int4(q, stream)
    ki, ks = quantize_int4(k, stream)
    vi, vs = quantize_int8(v, True, stream)
    o = torch.empty((B, H, Nq, d), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    attn_fwd_int8(qi, qs, ki, ks, vi, vs, o, lse, causal, scale, stream)
    return o, lse


def hadamard_signs(d: int, seed: int = 0, device="cuda"):
    """Seeded random sign vector (fp32, +-1) of the FP8 rotation H_d diag(signs)."""
    g = torch.Generator().manual_seed(int(seed))
    s = torch.randint(0, 2, (d,), generator=g, dtype=torch.int64) * 2 - 1
    return s.to(torch.float32).to(device)


def quantize_fp8(x: torch.Tensor, mode: int, signs: torch.Tensor | None = None, stream=None):
    """e4m3 codes (uint8) and fp32 scales of a bf16 [B,H,N,d] tensor: mode 0 per
    token row (rotated first when ``signs`` is given), mode 1 per channel."""
    B, H, N, d = x.shape
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scales = torch.empty((B, H, N) if mode == 0 else (B, H, d), dtype=torch.float32, device=x.device)
    attn_quantize_fp8(x, codes, scales, mode, signs, stream)
    return codes, scales


def forward_fp8(q, k, v, causal: bool = False, scale: float | None = None, rotate: bool = True,
                signs: torch.Tensor | None = None, stream=None):
    """Quantise bf16 q, k (per token, rotated by H_d diag(signs) unless
    ``rotate`` is False) and v (per channel) to e4m3 and run the FP8 forward.
    Returns (o fp32, lse fp32)."""
    B, H, Nq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if rotate and signs is None:
        signs = hadamard_signs(d, 0, q.device)
    sg = signs if rotate else None
    qc, qs = quantize_fp8(q, 0, sg, stream)
    kc, ks = quantize_fp8(k, 0, sg, stream)
    vc, vs = quantize_fp8(v, 1, None, stream)
    o = torch.empty((B, H, Nq, d), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    attn_fwd_fp8(qc, qs, kc, ks, vc, vs, o, lse, causal, scale, rotate, stream)
    return o, lse


def quantize_nvfp4(x: torch.Tensor, mode: int, stream=None):
    """NVFP4 codes + tiled scales of a bf16 [B,H,N,128] tensor (mode 0: Q/K,
    mode 1: V, written transposed)."""
    B, H, N, d = x.shape
    codes = torch.empty(attn_nvfp4_codes_bytes(B, H, N, d, mode), dtype=torch.uint8, device=x.device)
    sf = torch.empty(attn_nvfp4_sf_bytes(B, H, N, d, mode), dtype=torch.uint8, device=x.device)
    attn_quantize_nvfp4(x, codes, sf, mode, stream)
    return codes, sf


def forward_fp4(q, k, v, causal: bool = False, scale: float | None = None, p_mode: int = DIRECT_P, stream=None):
    """Quantise bf16 q, k, v to NVFP4 and run the FP4 forward.  Returns (o fp32, lse fp32)."""
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    qc, qs = quantize_nvfp4(q, 0, stream)
    kc, ks = quantize_nvfp4(k, 0, stream)
    vc, vs = quantize_nvfp4(v, 1, stream)
    o = torch.empty((B, H, Nq, d), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    attn_fwd_fp4(qc, qs, kc, ks, vc, vs, o, lse, B, H, Nq, Nkv, causal, scale, p_mode, stream)
    return o, lse
