"""GPU parity of grouped-query / multi-query attention (attn_fwd_gqa,
attn_decode_gqa) against the fp64 oracle's grouped-query definition, through
the C ABI.  Same tolerances as the bf16 path (max-abs 2e-2, mean-abs 2e-3 on
O, 1e-3 on LSE)."""
import numpy as np
import pytest

from oracle import attention as A
from tests import _guard as G
from tests._parity import assert_bf16_close
from workloads import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


def gqa_inputs(name, seed, B, Hq, Hkv, Nq, Nkv, d, device="cpu"):
    q, k, v = make_qkv(name, seed=seed, device=device, B=B, H=Hq, Nq=Nq, Nkv=Nkv, d=d)
    return q, k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 8, 2, 300, 333, 128), (2, 4, 1, 129, 1000, 64), (1, 6, 3, 256, 256, 128),
                                   (1, 4, 2, 640, 200, 64), (2, 2, 2, 128, 128, 128)],
                         ids=lambda s: "x".join(map(str, s)))
def test_fwd_gqa(cuda_lib, shape, causal):
    B, Hq, Hkv, Nq, Nkv, d = shape
    q, k, v = gqa_inputs("prefill", 31, B, Hq, Hkv, Nq, Nkv, d)
    o, lse = G.forward(cuda_lib, q.cuda(), k.cuda(), v.cuda(), causal, d ** -0.5)
    assert cuda_lib.attn_check_status() == 0
    O, L = A.attention_gqa(q, k, v, causal, d ** -0.5)
    assert_bf16_close(o, lse, O, L, f"gqa {shape} causal={causal}")


def test_fwd_gqa_equals_expanded_heads(cuda_lib):
    """The grouped call gives the same bits as attn_fwd on K/V expanded to one
    head per query head (the same kernel path, only the head mapping differs)."""
    q, k, v = gqa_inputs("prefill", 5, 1, 8, 2, 512, 700, 128)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    idx = A.kv_head_index(8, 2).tolist()
    o1, l1 = cuda_lib.forward(q, k, v, False, 0.1)
    o2, l2 = cuda_lib.forward(q, k[:, idx].contiguous(), v[:, idx].contiguous(), False, 0.1)
    assert cuda_lib.attn_check_status() == 0
    assert bool((o1 == o2).all()) and bool((l1 == l2).all())


# (B, Hq, Hkv, Nkv, d, splits).  d = 128 runs the tensor-core kernel with G
# query heads per work item, G the largest divisor of the group <= 8: groups
# 4, 8, 3, 16 (two items per cache head), 5 and 7; chunks shorter than a 64-key
# tile, chunks with no key at all (splits > Nkv), one exact tile, and more
# items than CTAs (persistent CTAs take several).  d = 64 runs the CUDA-core
# kernel (groups of 8 -> CTAs of 4, 2 -> 2).
@pytest.mark.parametrize("shape", [(4, 32, 8, 3000, 128, 16), (2, 8, 1, 8192, 64, 7), (3, 6, 2, 100, 128, 16),
                                   (2, 6, 3, 2000, 64, 5), (1, 16, 2, 700, 128, 1), (1, 16, 1, 1000, 128, 4),
                                   (2, 10, 2, 513, 128, 3), (1, 7, 1, 64, 128, 2), (2, 8, 2, 5, 128, 16),
                                   (8, 32, 4, 4096, 128, 32)],
                         ids=lambda s: "x".join(map(str, s)))
def test_decode_gqa(cuda_lib, shape):
    B, Hq, Hkv, Nkv, d, splits = shape
    q, k, v = gqa_inputs("decode", 8, B, Hq, Hkv, 1, Nkv, d)
    o, lse = G.decode(cuda_lib, q.cuda(), k.cuda(), v.cuda(), d ** -0.5, splits)
    assert cuda_lib.attn_check_status() == 0
    O, L = A.attention_gqa(q, k, v, False, d ** -0.5)
    assert_bf16_close(o, lse, O, L, f"decode gqa {shape}")


def test_decode_gqa_full_size_sampled_heads(cuda_lib):
    """Decode workload shape with 4 query heads per cache head (B64 Hq32 Hkv8
    N_kv 8192 d128, 16 splits), the launch the benchmark times; the oracle
    checks sampled (batch, head) pairs."""
    w = WORKLOADS["decode"]
    q, k, v = gqa_inputs(w, 0, w.B, w.H, w.H // 4, 1, w.Nkv, w.d, device="cuda")
    o, lse = G.decode(cuda_lib, q, k, v, w.scale, w.num_splits)
    assert cuda_lib.attn_check_status() == 0
    g = np.random.default_rng(3)
    for b, h in [(0, 0), (w.B - 1, w.H - 1)] + [tuple(x) for x in g.integers(0, [w.B, w.H], size=(8, 2))]:
        kh = h // 4
        O, L = A.attention(q[b:b + 1, h:h + 1], k[b:b + 1, kh:kh + 1], v[b:b + 1, kh:kh + 1], False, w.scale)
        assert_bf16_close(o[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1], O, L, f"decode gqa b={b} h={h}")
