"""Seeded synthetic inputs and the shapes of the attention workloads.

This module is shared by the fp64 oracle tests, the GPU parity tests and the
benchmark.  It holds no attention arithmetic: it only draws numbers and rounds
them to the storage type.  Everything the method computes lives in the oracle
(``oracle/``) and, independently, in the CUDA library.

Generator: one ``torch.Generator`` per call, seeded with the workload's seed;
Q, K and V are drawn in that order from the same stream as i.i.d. N(0, 1) fp32
values, multiplied (in fp32) by the workload's input scale and rounded to
bfloat16 with round-to-nearest-even.  On the CPU the stream is torch's
Mersenne-Twister normal sampler, on a CUDA device torch's Philox sampler; the
two streams differ, so a test that compares two implementations always hands
both the very same tensors.

Workloads (the shapes of the pages' examples; see ``WORKLOADS``):

* ``tiny``      B=1, H=2, N=128, d=64, scale 1/8
* ``prefill``   B=4, H=16, N=4096, d=128, scale 1/sqrt(128)
* ``longseq``   B=1, H=12, N=23400 (one 6.5 h trading day at 1 s), d=64,
                inputs x0.5, scale 1/8
* ``decode``    B=64, H=32, one query, N_kv=8192, d=128, 16 KV splits
* ``lowp``      B=2, H=24, N=8192, d=128, 4 outlier channels per head x20
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = ["Workload", "WORKLOADS", "normal_bf16", "make_qkv", "outlier_channels", "rotation_signs", "make_varlen"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Nq: int
    Nkv: int
    d: int
    scale: float
    input_scale: float = 1.0
    outliers_per_head: int = 0
    outlier_gain: float = 1.0
    num_splits: int = 1
    causal_modes: tuple = (False, True)
    note: str = field(default="", compare=False)

    def flops(self, causal: bool) -> float:
        """Algorithmic FLOPs of one forward: 4*B*H*Nq*Nkv*d, halved if causal."""
        f = 4.0 * self.B * self.H * self.Nq * self.Nkv * self.d
        return f / 2 if causal else f


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 128, 128, 64, 1.0 / 8.0,
                     note="correctness case, oracle in well under a second"),
    "prefill": Workload("prefill", 4, 16, 4096, 4096, 128, 1.0 / math.sqrt(128.0),
                        note="bf16 prefill, causal and non-causal"),
    "longseq": Workload("longseq", 1, 12, 23400, 23400, 64, 1.0 / 8.0, input_scale=0.5,
                        note="one trading day at 1 s resolution; 23400 = 182*128 + 104"),
    "decode": Workload("decode", 64, 32, 1, 8192, 128, 1.0 / math.sqrt(128.0),
                       num_splits=16, causal_modes=(False,),
                       note="memory-bound decode, split-KV into 16 chunks + combine"),
    "lowp": Workload("lowp", 2, 24, 8192, 8192, 128, 1.0 / math.sqrt(128.0),
                     outliers_per_head=4, outlier_gain=20.0, causal_modes=(False,),
                     note="INT8 / FP4 prefill with outlier channels"),
}


def normal_bf16(shape, gen: torch.Generator, device, input_scale: float = 1.0,
                channel_gain: torch.Tensor | None = None,
                chunk_elems: int = 1 << 28) -> torch.Tensor:
    """Draw i.i.d. N(0,1) fp32, multiply by ``input_scale`` (and by a per-(head,
    channel) gain broadcast over the last axis), round to bf16 (RNE).

    Drawn in chunks along the first axes so that very large tensors do not need
    a full fp32 temporary.
    """
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1, shape[-1]) if len(shape) > 1 else out.view(1, -1)
    rows_per_chunk = max(1, chunk_elems // flat.shape[1])
    gain_rows = None
    if channel_gain is not None:
        # channel_gain: [H, d]; rows of ``flat`` are ordered [B][H][N].
        B, H, N, d = shape
        gain_rows = channel_gain.to(device=device, dtype=torch.float32)
    for r0 in range(0, flat.shape[0], rows_per_chunk):
        r1 = min(flat.shape[0], r0 + rows_per_chunk)
        x = torch.randn((r1 - r0, flat.shape[1]), generator=gen, device=device,
                        dtype=torch.float32)
        if input_scale != 1.0:
            x.mul_(input_scale)
        if gain_rows is not None:
            B, H, N, d = shape
            head = (torch.arange(r0, r1, device=device) // N) % H
            x.mul_(gain_rows[head])
        flat[r0:r1].copy_(x.to(torch.bfloat16))
    return out


def outlier_channels(H: int, d: int, count: int, gen: torch.Generator) -> torch.Tensor:
    """Per head, ``count`` distinct channel indices (a seeded permutation prefix)."""
    return torch.stack([torch.randperm(d, generator=gen)[:count] for _ in range(H)])


def make_qkv(w: Workload | str, seed: int = 0, device="cpu", B: int | None = None,
             H: int | None = None, Nq: int | None = None, Nkv: int | None = None,
             d: int | None = None):
    """Q, K, V (bf16, [B][H][N][d], contiguous) for a workload, optionally with
    overridden sizes (used for small parity cases with the workload's value
    distribution).  Returns (q, k, v)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    B = w.B if B is None else B
    H = w.H if H is None else H
    Nq = w.Nq if Nq is None else Nq
    Nkv = w.Nkv if Nkv is None else Nkv
    d = w.d if d is None else d
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    gain = None
    if w.outliers_per_head:
        cpu_gen = torch.Generator()
        cpu_gen.manual_seed(seed + 1_000_003)
        idx = outlier_channels(H, d, w.outliers_per_head, cpu_gen)
        gain = torch.ones(H, d, dtype=torch.float32)
        gain.scatter_(1, idx, w.outlier_gain)
    q = normal_bf16((B, H, Nq, d), gen, dev, w.input_scale, gain)
    k = normal_bf16((B, H, Nkv, d), gen, dev, w.input_scale, gain)
    v = normal_bf16((B, H, Nkv, d), gen, dev, w.input_scale, gain)
    return q, k, v


def rotation_signs(d: int, seed: int = 0) -> torch.Tensor:
    """Seeded random sign vector (fp32 +-1, CPU) for the FP8 path's rotation:
    d Bernoulli(1/2) draws of a torch CPU generator, mapped {0, 1} -> {-1, +1}.
    The rotation draws these numbers; both implementations receive them."""
    g = torch.Generator()
    g.manual_seed(seed + 7_000_003)
    return (torch.randint(0, 2, (d,), generator=g, dtype=torch.int64) * 2 - 1).to(torch.float32)


def make_varlen(lens_q, lens_k, H: int, Hkv: int, d: int, seed: int = 0, input_scale: float = 1.0):
    """A variable-length batch packed without padding: q [sum(lens_q)][H][d],
    k, v [sum(lens_k)][Hkv][d] (bf16, drawn like ``normal_bf16``, in that
    order) and the int32 offset arrays cu_q, cu_k ([B + 1], starting at 0).
    Returns (q, k, v, cu_q, cu_k) on the CPU."""
    gen = torch.Generator()
    gen.manual_seed(seed + 9_000_011)
    tq, tk = int(sum(lens_q)), int(sum(lens_k))
    q = normal_bf16((tq, H, d), gen, "cpu", input_scale)
    k = normal_bf16((tk, Hkv, d), gen, "cpu", input_scale)
    v = normal_bf16((tk, Hkv, d), gen, "cpu", input_scale)
    cu_q = torch.tensor([0] + list(torch.cumsum(torch.tensor(lens_q), 0).tolist()), dtype=torch.int32)
    cu_k = torch.tensor([0] + list(torch.cumsum(torch.tensor(lens_k), 0).tolist()), dtype=torch.int32)
    return q, k, v, cu_q, cu_k
