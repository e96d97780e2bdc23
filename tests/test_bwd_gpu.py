"""GPU parity of attn_bwd (bf16 backward by recomputation) against the fp64
oracle's gradients, through the C ABI.

The device computes with bf16 operands: O from the device forward, P and dS
rounded to bf16 before their MMAs, bf16 outputs.  Each rounding is a relative
2^-9; the tolerance is 2^-7 of the largest reference magnitude of the tensor
(max-abs) and 2^-9 of its mean magnitude plus that (mean-abs), per gradient.
"""
import numpy as np
import pytest
import torch

from oracle import attention as A
from tests import _guard as G
from workloads import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


def _grads(ta, q, k, v, do, causal, scale):
    q, k, v, do = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = G.forward(ta, q, k, v, causal, scale)
    dq, dk, dv = G.backward(ta, q, k, v, o, lse, do, causal, scale)
    assert ta.attn_check_status() == 0
    return [t.double().cpu().numpy() for t in (dq, dk, dv)]


def _check(got, ref, what):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.isfinite(g).all(), f"{what} {name}: non-finite"
        err = np.abs(g - r)
        big = float(np.abs(r).max(initial=0.0))
        mean = float(np.abs(r).mean()) if r.size else 0.0
        print(f"{what} {name}: max err {err.max(initial=0):.3e} (ref max {big:.3e}), "
              f"mean err {err.mean() if err.size else 0:.3e} (ref mean {mean:.3e})")
        assert err.max(initial=0.0) <= 2.0 ** -7 * big + 1e-6, f"{what} {name}"
        assert (err.mean() if err.size else 0.0) <= 2.0 ** -9 * mean + 2.0 ** -7 * big / 64 + 1e-7, f"{what} {name}"


SHAPES = [
    # B, H, Nq, Nkv, d
    (1, 2, 128, 128, 64),
    (1, 1, 300, 333, 128),
    (2, 1, 129, 1000, 64),
    (1, 1, 640, 200, 128),     # causal: the first rows see no key
    (1, 2, 384, 384, 128),
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_backward_small(cuda_lib, shape, causal):
    B, H, Nq, Nkv, d = shape
    q, k, v = make_qkv("prefill", seed=41, B=B, H=H, Nq=Nq, Nkv=Nkv, d=d)
    do = make_qkv("prefill", seed=42, B=B, H=H, Nq=Nq, Nkv=1, d=d)[0]
    scale = d ** -0.5
    got = _grads(cuda_lib, q, k, v, do, causal, scale)
    ref = A.attention_backward(q, k, v, do, causal, scale)
    _check(got, ref, f"{shape} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_backward_prefill_workload_sampled_heads(cuda_lib, causal):
    """The prefill workload shape (B4 H16 N4096 d128); the oracle checks two
    (batch, head) slices (heads are independent)."""
    w = WORKLOADS["prefill"]
    q, k, v = make_qkv(w, seed=0)
    do = make_qkv(w, seed=1, Nkv=1)[0]
    got = _grads(cuda_lib, q, k, v, do, causal, w.scale)
    for b, h in [(0, 0), (3, 15)]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        ref = A.attention_backward(q[sl], k[sl], v[sl], do[sl], causal, w.scale)
        _check([g[sl] for g in got], ref, f"prefill b={b} h={h} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 2, 128, 128, 64), (1, 1, 300, 333, 128), (1, 1, 640, 200, 128),
                                   (1, 2, 384, 384, 128)], ids=lambda s: "x".join(map(str, s)))
def test_backward_fp8_p(cuda_lib, shape, causal):
    """FP8-P backward: dQ, dK as the bf16 backward; dV against the oracle with
    P rounded to e4m3, checked against the interval of dV over both roundings
    of every P element within fp32 evaluation error (relative 2e-5) of an
    e4m3 midpoint (dV is linear in the rounded P).  O and LSE are the oracle's
    (rounded to bf16 / fp32), so the device recomputes P from the same
    statistics."""
    from oracle import fp8 as F
    B, H, Nq, Nkv, d = shape
    q, k, v = make_qkv("prefill", seed=51, B=B, H=H, Nq=Nq, Nkv=Nkv, d=d)
    do = make_qkv("prefill", seed=52, B=B, H=H, Nq=Nq, Nkv=1, d=d)[0]
    scale = d ** -0.5
    O, L = A.attention(q, k, v, causal, scale)
    o = torch.from_numpy(O).to(torch.bfloat16).cuda()
    lse = torch.from_numpy(L).to(torch.float32).cuda()
    dq, dk, dv = G.backward(cuda_lib, q.cuda(), k.cuda(), v.cuda(), o, lse, do.cuda(), causal, scale, p_fp8=True)
    assert cuda_lib.attn_check_status() == 0
    got = [t.double().cpu().numpy() for t in (dq, dk, dv)]
    rq, rk, rv, (lo, hi) = A.attention_backward(q, k, v, do, causal, scale, p_round=F.e4m3_encode_value,
                                                p_grid=F.UE4M3_VALUES, p_rel=2e-5)
    _check(got[:2], (rq, rk), f"fp8p {shape} causal={causal}")
    big = float(np.abs(rv).max())
    tol = 2.0 ** -7 * big + 1e-6
    outside = np.maximum(np.maximum(lo - got[2], got[2] - hi), 0.0)
    n_flag = int(np.count_nonzero(hi - lo))
    print(f"fp8p {shape} causal={causal} dv: max err vs the oracle's rounding {np.abs(got[2] - rv).max():.3e}, "
          f"outside the interval of admissible roundings {outside.max():.3e} (tol {tol:.3e}, ref max {big:.3e}), "
          f"dV elements touched by a flagged P {n_flag}, widest interval {(hi - lo).max():.3e}")
    assert outside.max() <= tol
    # the 8-bit P moves dV away from the exact gradient by far more than the bf16 path does
    _, _, dv_exact = A.attention_backward(q, k, v, do, causal, scale)
    assert np.abs(rv - dv_exact).max() > 0
