"""GPU parity of the variable-length (packed) forward and of decode with a
cache length per batch entry against the fp64 oracle, through the C ABI.  Same
tolerances as the bf16 path (max-abs 2e-2, mean-abs 2e-3 on O, 1e-3 on LSE).
Outputs and workspaces sit between guard bands (tests._guard): the varlen
epilogue stores rows directly, so a row past its sequence would land in the
next sequence's rows or past the packed tensor."""
import pytest
import torch

from oracle import attention as A
from tests import _guard as G
from tests._parity import assert_bf16_close
from workloads import make_qkv, make_varlen

pytestmark = pytest.mark.gpu

MIXES = {
    "ragged": ([5, 0, 130, 300, 1, 257], [7, 4, 130, 100, 1, 700]),
    "tile_edges": ([127, 128, 129, 255, 256, 257], [128, 127, 129, 256, 255, 511]),
    "no_keys": ([64, 200], [0, 190]),
    "single": ([700], [900]),
}


def _run(ta, lq, lk, H, Hkv, d, causal, seed=0):
    q, k, v, cu_q, cu_k = make_varlen(lq, lk, H, Hkv, d, seed)
    o, lse = G.forward_varlen(ta, q.cuda(), k.cuda(), v.cuda(), cu_q.cuda(), cu_k.cuda(), max(lq), causal, d ** -0.5)
    assert ta.attn_check_status() == 0
    O, L = A.attention_varlen(q, k, v, cu_q.numpy(), cu_k.numpy(), causal, d ** -0.5)
    return o, lse, O, L, (q, k, v, cu_q, cu_k)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mix", sorted(MIXES))
def test_varlen_forward(cuda_lib, mix, d, causal):
    lq, lk = MIXES[mix]
    o, lse, O, L, _ = _run(cuda_lib, lq, lk, 4, 4, d, causal, seed=len(mix))
    assert_bf16_close(o, lse, O, L, f"varlen {mix} d={d} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_forward_grouped_query(cuda_lib, causal):
    o, lse, O, L, _ = _run(cuda_lib, [300, 129, 1000], [333, 500, 1000], 8, 2, 128, causal, seed=3)
    assert_bf16_close(o, lse, O, L, f"varlen gqa causal={causal}")


def test_varlen_equal_lengths_match_the_dense_kernel_bitwise(cuda_lib):
    """Equal lengths: the packed call runs the same tiles as attn_fwd on the
    [B][H][N][d] layout; rows of a neighbouring sequence that enter a ragged
    tile are masked, so the two give the same bits."""
    B, H, N, d = 3, 4, 333, 128
    q, k, v, cu_q, cu_k = make_varlen([N] * B, [N] * B, H, H, d, seed=7)
    for causal in (False, True):
        o, lse = cuda_lib.forward_varlen(q.cuda(), k.cuda(), v.cuda(), cu_q.cuda(), cu_k.cuda(), N, causal, 0.1)
        dense = [t.view(B, N, H, d).transpose(1, 2).contiguous().cuda() for t in (q, k, v)]
        od, ld = cuda_lib.forward(*dense, causal, 0.1)
        assert cuda_lib.attn_check_status() == 0
        assert torch.equal(o.view(B, N, H, d).transpose(1, 2).cpu(), od.cpu())
        assert torch.equal(lse.view(H, B, N).transpose(0, 1).cpu(), ld.cpu())


def test_varlen_longer_sequences_sampled(cuda_lib):
    lq = [4096, 1000, 2500]
    o, lse, O, L, _ = _run(cuda_lib, lq, lq, 4, 4, 128, True, seed=5)
    assert_bf16_close(o, lse, O, L, "varlen long causal")


@pytest.mark.parametrize("Hkv", [8, 2])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_varlen(cuda_lib, d, Hkv):
    B, H, N = 5, 8, 3000
    q, k, v = make_qkv("decode", seed=8, B=B, H=H, Nkv=N, d=d)
    k, v = k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()
    lens = torch.tensor([3000, 0, 1, 1234, 129], dtype=torch.int32)
    o, lse = G.decode_varlen(cuda_lib, q.cuda(), k.cuda(), v.cuda(), lens.cuda(), d ** -0.5, 16)
    assert cuda_lib.attn_check_status() == 0
    O, L = A.decode_varlen(q, k, v, lens.numpy(), d ** -0.5)
    assert_bf16_close(o, lse, O, L, f"decode varlen d={d} Hkv={Hkv}")


def test_decode_varlen_full_lengths_match_decode_bitwise(cuda_lib):
    q, k, v = make_qkv("decode", seed=9, B=3, H=4, Nkv=2048, d=128)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    lens = torch.full((3,), 2048, dtype=torch.int32, device="cuda")
    o1, l1 = cuda_lib.decode_varlen(q, k, v, lens, 0.1, num_splits=8)
    o2, l2 = cuda_lib.decode(q, k, v, 0.1, num_splits=8)
    assert cuda_lib.attn_check_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
