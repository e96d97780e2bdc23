"""GPU parity of the INT8 path against the oracle, through the C ABI.

* quantisers: bit-exact (codes and fp32 scales) against the oracle's fp32
  quantisers;
* int32 score tiles of the INT8 tensor-core path: bit-exact against the exact
  integer product;
* forward: within 5e-3 max-abs of the oracle's step-by-step INT8 emulation.
  Where an element of 127 * 2^(x - m) lies within fp32 evaluation error of a
  rounding midpoint the device may round it either way; the oracle then gives
  the interval of outputs over both roundings (``oracle.outcomes``) and the
  device must lie within 5e-3 of it.  Flagged rows and elements are reported
  and bounded.

Every output sits between guard bands that must survive the call
(``tests._guard``).
"""
import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import lowp as Q
from tests import _guard as G
from tests._parity import assert_within_outcomes, visible_scores
from workloads import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().numpy()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("name", ["prefill", "lowp"])
def test_quantisers_bit_exact(cuda_lib, name, d):
    q, k, v = make_qkv(name, seed=4, B=2, H=3, Nq=257, Nkv=130, d=d)
    q[0, 1, 7] = 0                                    # an all-zero row
    qg = q.cuda()
    xq, xs = G.quantize_int8(cuda_lib, qg, per_head=False)
    rq, rs = Q.quantize_int8_rows(q)
    assert np.array_equal(_np(xq), rq) and np.array_equal(_np(xs), rs)
    vq, vsc = G.quantize_int8(cuda_lib, v.cuda(), per_head=True)
    rvq, rvs = Q.quantize_int8_heads(v)
    assert np.array_equal(_np(vq), rvq) and np.array_equal(_np(vsc), rvs)


@pytest.mark.parametrize("Nq,Nkv", [(128, 128), (200, 300), (1, 1), (513, 129)])
def test_int8_scores_bit_exact(cuda_lib, Nq, Nkv):
    g = torch.Generator().manual_seed(Nq * 1000 + Nkv)
    qi = torch.randint(-127, 128, (1, 2, Nq, 128), generator=g, dtype=torch.int8)
    ki = torch.randint(-127, 128, (1, 2, Nkv, 128), generator=g, dtype=torch.int8)
    s = G.Guarded((1, 2, Nq, Nkv), torch.int32)
    cuda_lib.attn_int8_scores(qi.cuda(), ki.cuda(), s.t)
    assert cuda_lib.attn_check_status() == 0
    s.check("attn_int8_scores")
    assert np.array_equal(_np(s.t), Q.int8_scores(qi.numpy(), ki.numpy()))


def _check_int8(ta, q, k, v, causal, scale, rows=None, what="", int4=False):
    """The device quantises and runs the forward; the oracle quantises the same
    bf16 inputs itself (its quantisers are bit-exact with the device's, checked
    separately) and emulates the forward."""
    qi, qs = G.quantize_int8(ta, q.cuda(), False, int4=int4)
    ki, ks = G.quantize_int8(ta, k.cuda(), False, int4=int4)
    vi, vs = G.quantize_int8(ta, v.cuda(), True)
    B, H, Nq, d = q.shape
    o, lse = G.fwd_int8(ta, qi, qs, ki, ks, vi, vs, causal, scale, what)
    assert ta.attn_check_status() == 0
    quant = Q.quantize_int4_rows if int4 else Q.quantize_int8_rows
    rqi, rqs = quant(q)
    rki, rks = quant(k)
    rvi, rvs = Q.quantize_int8_heads(v)
    O, L, R = Q.attention_int8(rqi, rqs, rki, rks, rvi, rvs, causal, scale, outcomes=True, rows=rows)
    og, lg = _np(o).astype(np.float64), _np(lse).astype(np.float64)
    if rows is not None:
        og, lg = og[:, :, rows], lg[:, :, rows]
    n_scores = B * H * visible_scores(Nq, k.shape[2], causal, rows)
    err, _ = assert_within_outcomes(og, lg, O, L, R, what, n_scores)
    # drift from the unquantised fp64 attention (reported, not bounded here)
    Oe, _ = A.attention(q, k, v, causal, scale, rows=rows)
    cos = float((og * Oe).sum() / (np.linalg.norm(og) * np.linalg.norm(Oe) + 1e-300))
    return err, R.flips, cos


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 2, 128, 128), (1, 1, 300, 333), (2, 2, 129, 1000), (1, 1, 1, 1),
                                   (1, 1, 640, 200)], ids=lambda s: "x".join(map(str, s)))
def test_int8_forward_small(cuda_lib, shape, causal):
    B, H, Nq, Nkv = shape
    q, k, v = make_qkv("prefill", seed=9, B=B, H=H, Nq=Nq, Nkv=Nkv, d=128)
    _check_int8(cuda_lib, q, k, v, causal, 128 ** -0.5, what=f"{shape} causal={causal}")


def test_int8_forward_outlier_inputs(cuda_lib):
    q, k, v = make_qkv("lowp", seed=1, B=1, H=4, Nq=1024, Nkv=1024)
    _, flips, cos = _check_int8(cuda_lib, q, k, v, False, 128 ** -0.5, what="lowp-dist")
    assert cos > 0.99


def test_int8_full_lowp_workload_sampled_rows(cuda_lib):
    w = WORKLOADS["lowp"]
    q, k, v = make_qkv(w, seed=0)
    rows = np.array(sorted({0, 1, 127, 128, 4095, 8190, 8191} | set(np.random.default_rng(0).choice(8192, 24).tolist())))
    _, flips, cos = _check_int8(cuda_lib, q, k, v, False, w.scale, rows=rows, what="lowp full")
    assert cos > 0.99


# ---------------------------------------------------------------- INT4 Q/K
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("name", ["prefill", "lowp"])
def test_int4_quantiser_bit_exact(cuda_lib, name, d):
    q, _, _ = make_qkv(name, seed=13, B=2, H=3, Nq=300, Nkv=1, d=d)
    q[0, 1, 7] = 0
    qi, qs = G.quantize_int8(cuda_lib, q.cuda(), False, int4=True)
    assert cuda_lib.attn_check_status() == 0
    rq, rs = Q.quantize_int4_rows(q)
    assert np.array_equal(_np(qi), rq) and np.array_equal(_np(qs), rs)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 2, 128, 128), (1, 1, 300, 333), (1, 1, 640, 200)],
                         ids=lambda s: "x".join(map(str, s)))
def test_int4_forward_small(cuda_lib, shape, causal):
    B, H, Nq, Nkv = shape
    q, k, v = make_qkv("prefill", seed=19, B=B, H=H, Nq=Nq, Nkv=Nkv, d=128)
    _, _, cos = _check_int8(cuda_lib, q, k, v, causal, 128 ** -0.5, what=f"int4 {shape} causal={causal}", int4=True)
    print(f"int4 {shape} causal={causal}: cosine vs fp64 {cos:.4f}")


def test_int4_full_lowp_workload_sampled_rows(cuda_lib):
    w = WORKLOADS["lowp"]
    q, k, v = make_qkv(w, seed=0)
    rows = np.array(sorted({0, 1, 127, 128, 8191} | set(np.random.default_rng(2).choice(8192, 11).tolist())))
    _, flips, cos = _check_int8(cuda_lib, q, k, v, False, w.scale, rows=rows, what="int4 lowp full", int4=True)
    print(f"int4 lowp: cosine vs fp64 {cos:.4f}, boundary elements {flips}")


def test_quantisers_exact_on_rounding_ties(cuda_lib):
    """Rows whose quotients x / s land exactly on half-integers (amax = 127 *
    2^k, so s = 2^k, and x = (j + 1/2) 2^k): every element is a rounding tie
    (round half to even), the case where a divide-free quotient could round
    the other way.  Codes and scales bit-exact against the oracle."""
    rows = []
    for k in range(-6, 7, 3):
        for sign in (1.0, -1.0):
            r = np.empty(128, dtype=np.float32)
            r[0] = 127.0 * 2.0 ** k
            j = np.arange(127)
            r[1:] = sign * (j + 0.5) * 2.0 ** k * np.where(j % 2, -1.0, 1.0)
            rows.append(r)
    x = torch.tensor(np.stack(rows)).reshape(1, 2, -1, 128).to(torch.bfloat16)
    assert torch.equal(x.float(), torch.tensor(np.stack(rows)).reshape(1, 2, -1, 128))  # exact in bf16
    xq, xs = G.quantize_int8(cuda_lib, x.cuda(), per_head=False)
    rq, rs = Q.quantize_int8_rows(x)
    assert np.array_equal(_np(xq), rq) and np.array_equal(_np(xs), rs)
    # per head: one scale 127 * 2^6 for each head, so ties only where x = (j + 1/2) 2^6
    vq, vsc = G.quantize_int8(cuda_lib, x.cuda(), per_head=True)
    rvq, rvs = Q.quantize_int8_heads(x)
    assert np.array_equal(_np(vq), rvq) and np.array_equal(_np(vsc), rvs)
