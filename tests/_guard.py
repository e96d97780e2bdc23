"""Guard bands around device outputs (the parity tests' out-of-bounds check).

Every output buffer a parity test hands to the library (O, LSE, packed varlen
O, quantiser codes and scales including the padded FP4 V^T layout, decode and
backward workspaces, gradients) is carved out of a larger allocation whose
head and tail -- ``GUARD`` bytes each, plus any rounding slack -- hold a
sentinel byte.  The interior starts as all-ones bytes (NaN in bf16/fp32), so an
output the kernel never wrote also fails the parity comparison.  After the
call the sentinels are compared byte for byte: a kernel that stores past
either end of a buffer fails the test even when its values are right.

The calls below mirror the package conveniences, with guarded buffers.
"""
from __future__ import annotations

import math

import torch

GUARD = 4096
SENTINEL = 0xA5
INTERIOR = 0xFF


class Guarded:
    """A contiguous device tensor of ``shape``/``dtype`` (or ``nbytes`` raw
    bytes) with sentinel guard bands on both sides."""

    def __init__(self, shape, dtype, device="cuda", nbytes=None, interior=INTERIOR):
        esize = torch.empty((), dtype=dtype).element_size()
        self.nbytes = int(nbytes) if nbytes is not None else esize * math.prod(shape)
        padded = -(-max(self.nbytes, 1) // 256) * 256
        self.raw = torch.full((GUARD + padded + GUARD,), SENTINEL, dtype=torch.uint8, device=device)
        self.raw[GUARD:GUARD + self.nbytes].fill_(interior)
        body = self.raw[GUARD:GUARD + self.nbytes]
        self.t = body.view(dtype).view(shape) if nbytes is None else body

    def check(self, what=""):
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.nbytes:]
        for name, part, base in (("before", head, 0), ("after", tail, GUARD + self.nbytes)):
            bad = torch.nonzero(part != SENTINEL)
            assert bad.numel() == 0, (f"{what}: {bad.numel()} guard bytes {name} the buffer were overwritten "
                                      f"(first at raw offset {base + int(bad[0])})")


def _done(ta, bufs, what):
    torch.cuda.synchronize()
    for b in bufs:
        b.check(what)


# ------------------------------------------------------------------ bf16 forward / decode
def forward(ta, q, k, v, causal, scale, what="attn_fwd"):
    B, H, Nq, d = q.shape
    o = Guarded((B, H, Nq, d), torch.bfloat16)
    lse = Guarded((B, H, Nq), torch.float32)
    if k.shape[1] != H:
        ta.attn_fwd_gqa(q, k, v, o.t, lse.t, causal, scale)
    else:
        ta.attn_fwd(q, k, v, o.t, lse.t, causal, scale)
    _done(ta, (o, lse), what)
    return o.t, lse.t


def decode(ta, q, k, v, scale, num_splits, what="attn_decode"):
    B, H, _, d = q.shape
    ws = Guarded(None, torch.uint8, nbytes=ta.attn_decode_workspace_bytes(B, H, d, num_splits))
    o = Guarded((B, H, 1, d), torch.bfloat16)
    lse = Guarded((B, H, 1), torch.float32)
    if k.shape[1] != H:
        ta.attn_decode_gqa(q, k, v, o.t, lse.t, scale, num_splits, ws.t)
    else:
        ta.attn_decode(q, k, v, o.t, lse.t, scale, num_splits, ws.t)
    _done(ta, (ws, o, lse), what)
    return o.t, lse.t


def decode_varlen(ta, q, k, v, seqlens, scale, num_splits, what="attn_decode_varlen"):
    B, H, _, d = q.shape
    ws = Guarded(None, torch.uint8, nbytes=ta.attn_decode_workspace_bytes(B, H, d, num_splits))
    o = Guarded((B, H, 1, d), torch.bfloat16)
    lse = Guarded((B, H, 1), torch.float32)
    ta.attn_decode_varlen(q, k, v, o.t, lse.t, seqlens, scale, num_splits, ws.t)
    _done(ta, (ws, o, lse), what)
    return o.t, lse.t


def forward_varlen(ta, q, k, v, cu_q, cu_k, max_seqlen_q, causal, scale, what="attn_fwd_varlen"):
    total_q, H, d = q.shape
    o = Guarded((total_q, H, d), torch.bfloat16)
    lse = Guarded((H, total_q), torch.float32)
    ta.attn_fwd_varlen(q, k, v, o.t, lse.t, cu_q, cu_k, max_seqlen_q, causal, scale)
    _done(ta, (o, lse), what)
    return o.t, lse.t


def backward(ta, q, k, v, o, lse, do, causal, scale, p_fp8=False, what="attn_bwd"):
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    dq = Guarded((B, H, Nq, d), torch.bfloat16)
    dk = Guarded((B, H, Nkv, d), torch.bfloat16)
    dv = Guarded((B, H, Nkv, d), torch.bfloat16)
    ws = Guarded(None, torch.uint8, nbytes=max(16, ta.attn_bwd_workspace_bytes(B, H, Nq)))
    (ta.attn_bwd_fp8p if p_fp8 else ta.attn_bwd)(q, k, v, o, do, lse, dq.t, dk.t, dv.t, causal, scale, ws.t)
    _done(ta, (dq, dk, dv, ws), what)
    return dq.t, dk.t, dv.t


# ------------------------------------------------------------------ quantised paths
def quantize_int8(ta, x, per_head, int4=False, what="attn_quantize_int8"):
    B, H, N, d = x.shape
    xq = Guarded((B, H, N, d), torch.int8)
    xs = Guarded((B, H) if per_head else (B, H, N), torch.float32)
    if int4:
        ta.attn_quantize_int4(x, xq.t, xs.t)
    else:
        ta.attn_quantize_int8(x, xq.t, xs.t, per_head)
    _done(ta, (xq, xs), what)
    return xq.t, xs.t


def fwd_int8(ta, qi, qs, ki, ks, vi, vs, causal, scale, what="attn_fwd_int8"):
    B, H, Nq, d = qi.shape
    o = Guarded((B, H, Nq, d), torch.float32)
    lse = Guarded((B, H, Nq), torch.float32)
    ta.attn_fwd_int8(qi, qs, ki, ks, vi, vs, o.t, lse.t, causal, scale)
    _done(ta, (o, lse), what)
    return o.t, lse.t


def quantize_nvfp4(ta, x, mode, what="attn_quantize_nvfp4"):
    B, H, N, d = x.shape
    codes = Guarded(None, torch.uint8, nbytes=ta.attn_nvfp4_codes_bytes(B, H, N, d, mode))
    sf = Guarded(None, torch.uint8, nbytes=ta.attn_nvfp4_sf_bytes(B, H, N, d, mode))
    ta.attn_quantize_nvfp4(x, codes.t, sf.t, mode)
    _done(ta, (codes, sf), what)
    return codes.t, sf.t


def forward_fp4(ta, q, k, v, causal, scale, p_mode, what="attn_fwd_fp4"):
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    qc, qs = quantize_nvfp4(ta, q, 0, what + " quantise q")
    kc, ks = quantize_nvfp4(ta, k, 0, what + " quantise k")
    vc, vs = quantize_nvfp4(ta, v, 1, what + " quantise v")
    o = Guarded((B, H, Nq, d), torch.float32)
    lse = Guarded((B, H, Nq), torch.float32)
    ta.attn_fwd_fp4(qc, qs, kc, ks, vc, vs, o.t, lse.t, B, H, Nq, Nkv, causal, scale, p_mode)
    _done(ta, (o, lse), what)
    return o.t, lse.t


def quantize_fp8(ta, x, mode, signs=None, what="attn_quantize_fp8"):
    B, H, N, d = x.shape
    codes = Guarded((B, H, N, d), torch.uint8)
    sc = Guarded((B, H, N) if mode == 0 else (B, H, d), torch.float32)
    ta.attn_quantize_fp8(x, codes.t, sc.t, mode, signs)
    _done(ta, (codes, sc), what)
    return codes.t, sc.t


def fwd_fp8(ta, qc, qs, kc, ks, vc, vs, causal, scale, rotated, what="attn_fwd_fp8"):
    B, H, Nq, d = qc.shape
    o = Guarded((B, H, Nq, d), torch.float32)
    lse = Guarded((B, H, Nq), torch.float32)
    ta.attn_fwd_fp8(qc, qs, kc, ks, vc, vs, o.t, lse.t, causal, scale, rotated)
    _done(ta, (o, lse), what)
    return o.t, lse.t
