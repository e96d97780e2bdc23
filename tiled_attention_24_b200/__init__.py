"""Fused tiled attention forward for NVIDIA B200 (sm_100a).

The compute lives in ``libtiledattn.so`` (CUDA kernels behind a C ABI, see
``include/tiledattn.h``); this package is its thin ctypes binding plus a few
conveniences that allocate outputs with torch and call the same entry points.
"""
from __future__ import annotations

import math

import torch

from ._binding import (AttnError, LIB_PATH, attn_check_status, attn_decode,  # noqa: F401
                       attn_decode_workspace_bytes, attn_fwd, attn_set_wait_limit_ns,
                       attn_status_string, attn_version, attn_watchdog_selftest, load)

__all__ = ["load", "attn_fwd", "attn_decode", "attn_decode_workspace_bytes", "attn_check_status",
           "attn_set_wait_limit_ns", "attn_watchdog_selftest", "attn_version", "attn_status_string",
           "AttnError", "forward", "decode"]


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
            scale: float | None = None, stream=None):
    """Allocate O (bf16) and LSE (fp32) and run ``attn_fwd``."""
    B, H, Nq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    attn_fwd(q, k, v, o, lse, causal, scale, stream)
    return o, lse


def decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
           num_splits: int = 16, workspace: torch.Tensor | None = None, stream=None):
    """Allocate O, LSE (and a workspace if none is given) and run ``attn_decode``."""
    B, H, _, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if workspace is None:
        nbytes = attn_decode_workspace_bytes(B, H, d, num_splits)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, 1), dtype=torch.float32, device=q.device)
    attn_decode(q, k, v, o, lse, scale, num_splits, workspace, stream)
    return o, lse
