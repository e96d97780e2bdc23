"""GPU parity of attn_fwd (bf16) against the fp64 oracle, through the C ABI.

Small cases run the oracle on every output; the full workloads (prefill
B4 H16 N4096 d128; long sequence B1 H12 N23400 d64) are checked on sampled
query rows of every head, in the same launch configuration the benchmark
times.  Tolerances: max-abs 2e-2, mean-abs 2e-3 on O, 1e-3 on LSE.
"""
import numpy as np
import pytest
import torch

from oracle import attention as A
from tests._parity import assert_bf16_close, to64
from workloads import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


def run(ta, q, k, v, causal, scale):
    o, lse = ta.forward(q.cuda(), k.cuda(), v.cuda(), causal, scale)
    assert ta.attn_check_status() == 0
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_workload(cuda_lib, causal):
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w, seed=0)
    o, lse = run(cuda_lib, q, k, v, causal, w.scale)
    O, L = A.attention(q, k, v, causal, w.scale)
    assert_bf16_close(o, lse, O, L, f"tiny causal={causal}")


RAGGED = [
    # B, H, Nq, Nkv, d
    (1, 1, 1, 1, 64),
    (1, 1, 1, 1, 128),
    (1, 2, 127, 127, 64),
    (2, 1, 129, 300, 128),
    (1, 1, 300, 129, 128),      # Nq > Nkv: causal rows before the diagonal see nothing
    (1, 3, 257, 513, 64),
    (1, 1, 384, 384, 128),
    (2, 2, 1000, 1000, 128),
    (1, 2, 640, 2000, 64),
    (1, 1, 200, 1, 64),
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", RAGGED, ids=lambda s: "x".join(map(str, s)))
def test_ragged_shapes(cuda_lib, shape, causal):
    B, H, Nq, Nkv, d = shape
    q, k, v = make_qkv("prefill", seed=11, B=B, H=H, Nq=Nq, Nkv=Nkv, d=d)
    scale = d ** -0.5
    o, lse = run(cuda_lib, q, k, v, causal, scale)
    O, L = A.attention(q, k, v, causal, scale)
    assert_bf16_close(o, lse, O, L, f"{shape} causal={causal}")


def test_causal_future_keys_do_not_matter(cuda_lib):
    q, k, v = make_qkv("prefill", seed=3, B=1, H=2, Nq=384, Nkv=384, d=128)
    o1, l1 = run(cuda_lib, q, k, v, True, 128 ** -0.5)
    k2, v2 = k.clone(), v.clone()
    k2[:, :, 200:] = torch.randn_like(k2[:, :, 200:].float()).mul(30).to(torch.bfloat16)
    v2[:, :, 200:] = torch.randn_like(v2[:, :, 200:].float()).mul(30).to(torch.bfloat16)
    o2, l2 = run(cuda_lib, q, k2, v2, True, 128 ** -0.5)
    assert torch.equal(o1[:, :, :200], o2[:, :, :200])
    assert torch.equal(l1[:, :, :200], l2[:, :, :200])


def test_single_key_and_equal_scores(cuda_lib):
    q, k, v = make_qkv("prefill", seed=5, B=1, H=2, Nq=130, Nkv=1, d=64)
    o, lse = run(cuda_lib, q, k, v, False, 0.125)
    assert torch.equal(o.cpu(), v.expand_as(o).contiguous())
    q0 = torch.zeros(1, 2, 130, 64, dtype=torch.bfloat16)
    _, k, v = make_qkv("prefill", seed=6, B=1, H=2, Nq=130, Nkv=777, d=64)
    o, lse = run(cuda_lib, q0, k, v, False, 0.125)
    mean = v.double().mean(dim=2, keepdim=True).expand(1, 2, 130, 64).numpy()
    assert np.abs(to64(o) - mean).max() < 4e-3
    assert np.abs(to64(lse) - np.log(777.0)).max() < 1e-4


def test_empty_inputs(cuda_lib):
    q = torch.zeros(2, 3, 0, 64, dtype=torch.bfloat16, device="cuda")
    o, lse = cuda_lib.forward(q, q, q, False, 0.125)
    assert o.numel() == 0
    q = torch.randn(1, 2, 5, 64, device="cuda").to(torch.bfloat16)
    kv = torch.zeros(1, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    o, lse = cuda_lib.forward(q, kv, kv, False, 0.125)
    assert cuda_lib.attn_check_status() == 0
    assert (o == 0).all() and torch.isneginf(lse).all()


def _sample_rows(N, count, seed):
    g = np.random.default_rng(seed)
    rows = set(g.choice(N, size=min(N, count), replace=False).tolist())
    rows |= {0, 1, 127, 128, 255, 256, N - 1, N - 2, N - 129}
    return np.array(sorted(r for r in rows if 0 <= r < N))


@pytest.mark.parametrize("name", ["prefill", "longseq"])
@pytest.mark.parametrize("causal", [False, True])
def test_full_workload_sampled_rows(cuda_lib, name, causal):
    w = WORKLOADS[name]
    q, k, v = make_qkv(w, seed=0)
    o, lse = run(cuda_lib, q, k, v, causal, w.scale)
    rows = _sample_rows(w.Nq, 48, 99)
    O, L = A.attention(q, k, v, causal, w.scale, rows=rows)
    assert_bf16_close(o[:, :, rows], lse[:, :, rows], O, L, f"{name} causal={causal}")
    assert torch.isfinite(lse).all()


def test_repeated_calls_are_deterministic(cuda_lib):
    q, k, v = make_qkv("prefill", seed=8, B=2, H=4, Nq=1024, Nkv=1024, d=128)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = cuda_lib.forward(q, k, v, True, 128 ** -0.5)
    o2, l2 = cuda_lib.forward(q, k, v, True, 128 ** -0.5)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
