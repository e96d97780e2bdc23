"""GPU parity of attn_decode (split-KV + combine) against the fp64 oracle.
O, LSE and the split workspace sit between guard bands (tests._guard)."""
import numpy as np
import pytest
import torch

from oracle import attention as A
from tests import _guard as G
from tests._parity import assert_bf16_close
from workloads import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Nkv,splits", [(1, 1), (1, 16), (100, 16), (511, 1), (8192, 16), (3000, 7),
                                        (1200, 1024), (20000, 3)])
def test_decode_small(cuda_lib, d, Nkv, splits):
    q, k, v = make_qkv("decode", seed=2, B=2, H=3, Nq=1, Nkv=Nkv, d=d)
    scale = d ** -0.5
    o, lse = G.decode(cuda_lib, q.cuda(), k.cuda(), v.cuda(), scale, splits)
    assert cuda_lib.attn_check_status() == 0
    O, L = A.decode(q, k, v, scale)
    assert_bf16_close(o, lse, O, L, f"decode Nkv={Nkv} splits={splits}")


def test_split_count_does_not_change_the_result_beyond_rounding(cuda_lib):
    q, k, v = make_qkv("decode", seed=4, B=4, H=4, Nq=1, Nkv=4096, d=128)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    outs = [cuda_lib.decode(q, k, v, None, s) for s in (1, 2, 16, 64)]
    for o, lse in outs[1:]:
        assert (o.float() - outs[0][0].float()).abs().max().item() < 4e-3
        assert (lse - outs[0][1]).abs().max().item() < 1e-4


def test_full_decode_workload_sampled_heads(cuda_lib):
    w = WORKLOADS["decode"]
    q, k, v = make_qkv(w, seed=0, device="cuda")
    o, lse = G.decode(cuda_lib, q, k, v, w.scale, w.num_splits)
    assert cuda_lib.attn_check_status() == 0
    g = np.random.default_rng(0)
    for b, h in [(0, 0), (w.B - 1, w.H - 1)] + [tuple(x) for x in g.integers(0, [w.B, w.H], size=(10, 2))]:
        O, L = A.decode(q[b:b + 1, h:h + 1].cpu(), k[b:b + 1, h:h + 1].cpu(), v[b:b + 1, h:h + 1].cpu(), w.scale)
        assert_bf16_close(o[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1], O, L, f"decode b={b} h={h}")
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
