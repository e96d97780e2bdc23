"""Pins of the fp64 oracle (bf16 path and decode) to facts fixed outside it.

Closed forms, invariants, an independent library routine (PyTorch's fp64
scaled_dot_product_attention on the CPU, the drop-in named by the
Flash Attention trading-models page, "Integration in eight lines"), brute force
on tiny inputs, and the pages' own blockwise algorithm.  No GPU.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A

RNG = np.random.default_rng(1234)


def rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def test_single_key_gives_that_value_row():
    q, k, v = rand(2, 3, 5, 8), rand(2, 3, 1, 8), rand(2, 3, 1, 8)
    O, L = A.attention(q, k, v, False, 0.3)
    assert np.array_equal(O, np.broadcast_to(v, O.shape))
    np.testing.assert_allclose(L, 0.3 * np.einsum("bhid,bhjd->bhi", q, k), rtol=0, atol=1e-14)


def test_equal_scores_give_mean_of_values():
    q = np.zeros((1, 2, 4, 16))
    k, v = rand(1, 2, 37, 16), rand(1, 2, 37, 16)
    O, L = A.attention(q, k, v, False, 0.125)
    np.testing.assert_allclose(O, np.broadcast_to(v.mean(axis=2, keepdims=True), O.shape),
                               rtol=0, atol=1e-14)
    np.testing.assert_allclose(L, math.log(37.0), rtol=0, atol=1e-14)


def test_causal_first_row_sees_only_first_key():
    q, k, v = rand(1, 2, 9, 4), rand(1, 2, 9, 4), rand(1, 2, 9, 4)
    O, L = A.attention(q, k, v, True, 0.5)
    np.testing.assert_array_equal(O[:, :, 0], v[:, :, 0])
    np.testing.assert_allclose(L[:, :, 0], 0.5 * (q[:, :, 0] * k[:, :, 0]).sum(-1), atol=1e-15)


def test_probability_rows_sum_to_one_and_mask_future():
    q, k = rand(1, 3, 11, 8, scale=3), rand(1, 3, 11, 8, scale=3)
    for causal in (False, True):
        P = A.softmax_rows(q, k, causal, 0.7)
        assert (P >= 0).all()
        np.testing.assert_allclose(P.sum(-1), 1.0, rtol=0, atol=1e-12)
        if causal:
            assert (P[..., np.triu_indices(11, 1)[0], np.triu_indices(11, 1)[1]] == 0).all()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nkv,d", [(1, 1, 1), (5, 7, 3), (7, 5, 3), (33, 70, 16), (64, 64, 64)])
def test_matches_torch_sdpa_fp64(causal, Nq, Nkv, d):
    """Independent library routine.  torch's is_causal is top-left aligned; the
    oracle is bottom-right aligned, so causal cases use an explicit bool mask."""
    q, k, v = rand(2, 3, Nq, d), rand(2, 3, Nkv, d), rand(2, 3, Nkv, d)
    scale = 1.0 / math.sqrt(d)
    O, L = A.attention(q, k, v, causal, scale)
    tq, tk, tv = (torch.from_numpy(t) for t in (q, k, v))
    mask = None
    if causal:
        i = torch.arange(Nq)[:, None]
        j = torch.arange(Nkv)[None, :]
        mask = j <= i + (Nkv - Nq)
    dead = (mask is not None) and (~mask.any(dim=1)).any().item()
    if not dead:
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask,
                                                               scale=scale).numpy()
        np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)
    S = torch.einsum("bhid,bhjd->bhij", tq, tk) * scale
    if mask is not None:
        S = S.masked_fill(~mask, float("-inf"))
    np.testing.assert_allclose(L, torch.logsumexp(S, dim=-1).numpy(), rtol=0, atol=1e-12)


def test_fully_masked_rows_are_zero_with_minus_inf_lse():
    # Nq > Nkv with bottom-right alignment: the first Nq - Nkv rows see nothing.
    q, k, v = rand(1, 1, 6, 4), rand(1, 1, 3, 4), rand(1, 1, 3, 4)
    O, L = A.attention(q, k, v, True, 1.0)
    assert (O[0, 0, :3] == 0).all() and np.isneginf(L[0, 0, :3]).all()
    np.testing.assert_array_equal(O[0, 0, 3], v[0, 0, 0])


def test_brute_force_loops_tiny():
    q, k, v = rand(1, 1, 3, 2), rand(1, 1, 4, 2), rand(1, 1, 4, 2)
    scale = 0.9
    for causal in (False, True):
        O, L = A.attention(q, k, v, causal, scale)
        for i in range(3):
            w = []
            for j in range(4):
                if causal and j > i + 1:
                    continue
                w.append((j, math.exp(scale * sum(q[0, 0, i, c] * k[0, 0, j, c] for c in range(2)))))
            z = sum(e for _, e in w)
            for c in range(2):
                o = sum(e * v[0, 0, j, c] for j, e in w) / z
                assert abs(O[0, 0, i, c] - o) < 1e-13
            assert abs(L[0, 0, i] - math.log(z)) < 1e-13


def test_causal_future_perturbation_leaves_rows_unchanged():
    q, k, v = rand(1, 2, 16, 8), rand(1, 2, 16, 8), rand(1, 2, 16, 8)
    O, L = A.attention(q, k, v, True, 0.4)
    for i in (0, 5, 14):
        k2, v2 = k.copy(), v.copy()
        k2[:, :, i + 1:] = rand(1, 2, 15 - i, 8, scale=50)
        v2[:, :, i + 1:] = rand(1, 2, 15 - i, 8, scale=50)
        O2, L2 = A.attention(q, k2, v2, True, 0.4)
        assert np.array_equal(O2[:, :, :i + 1], O[:, :, :i + 1])
        assert np.array_equal(L2[:, :, :i + 1], L[:, :, :i + 1])


def test_key_shift_and_permutation_invariance():
    q, k, v = rand(1, 2, 8, 6), rand(1, 2, 13, 6), rand(1, 2, 13, 6)
    O, L = A.attention(q, k, v, False, 0.3)
    c = rand(6)
    O2, L2 = A.attention(q, k + c, v, False, 0.3)
    np.testing.assert_allclose(O2, O, atol=1e-12)
    np.testing.assert_allclose(L2, L + 0.3 * q @ c, atol=1e-12)
    perm = RNG.permutation(13)
    O3, L3 = A.attention(q, k[:, :, perm], v[:, :, perm], False, 0.3)
    np.testing.assert_allclose(O3, O, atol=1e-13)
    np.testing.assert_allclose(L3, L, atol=1e-13)


def _adversarial(N, d):
    """Scores that grow block after block (every block raises the max) mixed
    with +-1e3 magnitudes."""
    q = rand(1, 1, N, d)
    k = rand(1, 1, N, d)
    k *= np.linspace(0.1, 30, N)[None, None, :, None]
    k[0, 0, N // 2] *= 1e3 / max(1.0, np.abs(k[0, 0, N // 2]).max())
    return q, k, rand(1, 1, N, d)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Br,Bc", [(1, 1), (2, 3), (3, 2), (4, 9), (9, 9)])
def test_pages_blockwise_algorithm_equals_definition(causal, Br, Bc):
    q, k, v = _adversarial(9, 3)
    O, L = A.attention(q, k, v, causal, 0.8)
    Ob, Lb = A.attention_blockwise(q, k, v, causal, 0.8, Br, Bc)
    np.testing.assert_allclose(Ob, O, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Lb, L, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Bc", [1, 2, 3, 9])
@pytest.mark.parametrize("tau", [0.0, 8.0])
def test_lazy_rescale_equals_definition(causal, Bc, tau):
    q, k, v = _adversarial(9, 3)
    O, L = A.attention(q, k, v, causal, 0.8)
    Ol, Ll = A.attention_lazy_rescale(q, k, v, causal, 0.8, Bc, tau)
    np.testing.assert_allclose(Ol, O, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Ll, L, rtol=1e-12, atol=1e-12)


def test_lazy_rescale_moves_the_reference_less_often():
    q, k, v = rand(1, 2, 256, 32), rand(1, 2, 1024, 32), rand(1, 2, 1024, 32)
    *_, r0 = A.attention_lazy_rescale(q, k, v, False, 1 / math.sqrt(32), 64, 0.0, True)
    *_, r8 = A.attention_lazy_rescale(q, k, v, False, 1 / math.sqrt(32), 64, 8.0, True)
    assert r8 < r0 and r8 == 0


def test_lazy_rescale_per_row_moves_and_margins_by_hand():
    """d = 1, q = 1, scale = ln 2 (so the base-2 logit of key j is k_j), blocks
    of 2 keys.  Row maxima per block 0, 10, 15, 30: the reference starts at 0,
    moves at block 1 (10 > 0 + 8, gap 2), stays at block 2 (15 < 10 + 8, gap
    3), moves at block 3 (30 > 18, gap 12): two moves, margin 2."""
    q = np.ones((1, 1, 1, 1))
    k = np.array([0.0, -1.0, 10.0, 4.0, 15.0, 2.0, 30.0, 29.0]).reshape(1, 1, 8, 1)
    v = np.arange(8.0).reshape(1, 1, 8, 1)
    O, L, moves, margin = A.attention_lazy_rescale(q, k, v, False, math.log(2.0), 2, 8.0, rescale_rows=True)
    assert moves[0, 0, 0] == 2 and abs(margin[0, 0, 0] - 2.0) < 1e-12
    *_, total = A.attention_lazy_rescale(q, k, v, False, math.log(2.0), 2, 8.0, True)
    assert total == 2
    O2, L2 = A.attention(q, k, v, False, math.log(2.0))
    np.testing.assert_allclose(O, O2, rtol=1e-12)


def test_lazy_rescale_per_row_moves_sum_to_the_total():
    q, k, v = rand(2, 2, 40, 8, scale=3.0), rand(2, 2, 70, 8, scale=3.0), rand(2, 2, 70, 8)
    for causal in (False, True):
        *_, total = A.attention_lazy_rescale(q, k, v, causal, 1.0, 8, 4.0, True)
        *_, moves, margin = A.attention_lazy_rescale(q, k, v, causal, 1.0, 8, 4.0, rescale_rows=True)
        assert moves.sum() == total and total > 0 and np.all(margin >= 0)


@pytest.mark.parametrize("splits", [1, 2, 3, 16, 40])
def test_split_kv_combine_equals_unsplit(splits):
    q, k, v = rand(3, 2, 1, 16), rand(3, 2, 37, 16), rand(3, 2, 37, 16)
    O, L = A.decode(q, k, v, 0.25)
    Op, Lp = A.decode_partials(q, k, v, 0.25, splits)
    Oc, Lc = A.combine(Op, Lp)
    np.testing.assert_allclose(Oc, O, rtol=0, atol=1e-13)
    np.testing.assert_allclose(Lc, L, rtol=0, atol=1e-13)


def test_split_bounds_cover_all_keys_once():
    for N, s in [(8192, 16), (37, 40), (1, 3), (100, 7)]:
        b = A.split_bounds(N, s)
        assert len(b) == s and b[0][0] == 0 and b[-1][1] == N
        assert all(b[i][1] == b[i + 1][0] for i in range(s - 1))


def test_bf16_inputs_convert_exactly():
    t = torch.randn(2, 2, 5, 8).to(torch.bfloat16)
    O, _ = A.attention(t, t, t, False, 0.1)
    O2, _ = A.attention(t.float().numpy().astype(np.float64), t.float().numpy(), t.float().numpy(),
                        False, 0.1)
    assert np.array_equal(O, O2)


# ---------------------------------------------------------------- GQA / MQA
@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 1), (6, 3), (3, 3)])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_matches_torch_sdpa_enable_gqa(Hq, Hkv, causal):
    """Pin against PyTorch's own grouped-query SDPA (fp64 on CPU), an
    implementation independent of the head-index substitution."""
    g = torch.Generator().manual_seed(Hq * 10 + Hkv)
    B, Nq, Nkv, d = 2, 7, 11 if not causal else 7, 5
    q = torch.randn(B, Hq, Nq, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, Nkv, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, Nkv, d, generator=g, dtype=torch.float64)
    O, _ = A.attention_gqa(q, k, v, causal, 0.4)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=0.4,
                                                           enable_gqa=True)
    assert np.abs(O - ref.numpy()).max() < 1e-12


def test_mqa_heads_share_one_kv_head():
    """Hkv = 1: every query head attends to the same keys and values, so two
    query heads with equal queries give equal outputs, and each head equals a
    single-head call with that head's queries."""
    g = torch.Generator().manual_seed(5)
    q = torch.randn(1, 4, 6, 8, generator=g, dtype=torch.float64)
    q[:, 3] = q[:, 1]
    k = torch.randn(1, 1, 9, 8, generator=g, dtype=torch.float64)
    v = torch.randn(1, 1, 9, 8, generator=g, dtype=torch.float64)
    O, L = A.attention_gqa(q, k, v, False, 0.3)
    assert np.array_equal(O[:, 3], O[:, 1]) and np.array_equal(L[:, 3], L[:, 1])
    for h in range(4):
        Oh, Lh = A.attention(q[:, h:h + 1], k, v, False, 0.3)
        assert np.array_equal(O[:, h:h + 1], Oh) and np.array_equal(L[:, h:h + 1], Lh)


def test_kv_head_index_groups_and_rejects_uneven():
    assert A.kv_head_index(8, 2).tolist() == [0, 0, 0, 0, 1, 1, 1, 1]
    assert A.kv_head_index(4, 4).tolist() == [0, 1, 2, 3]
    with pytest.raises(ValueError):
        A.kv_head_index(6, 4)


# ---------------------------------------------------------------- backward
@pytest.mark.parametrize("causal,Nq,Nkv", [(False, 7, 9), (True, 8, 8), (True, 5, 9), (True, 9, 4)])
def test_backward_matches_torch_autograd_fp64(causal, Nq, Nkv):
    """Pin against PyTorch autograd through its own fp64 attention (explicit
    scores, masked_fill, softmax, matmul): an implementation of the gradient
    independent of the closed-form expressions."""
    g = torch.Generator().manual_seed(Nq * 31 + Nkv)
    q, k, v, do = (torch.randn(2, 2, n, 5, generator=g, dtype=torch.float64) for n in (Nq, Nkv, Nkv, Nq))
    qr, kr, vr = (t.clone().requires_grad_(True) for t in (q, k, v))
    S = (qr @ kr.transpose(-1, -2)) * 0.35
    vis = torch.tensor(A.visible_mask(Nq, Nkv, causal))
    S = S.masked_fill(~vis, float("-inf"))
    P = torch.softmax(S, dim=-1).nan_to_num(0.0)      # rows with no visible key: P = 0
    (P @ vr).backward(do)
    dq, dk, dv = A.attention_backward(q, k, v, do, causal, 0.35)
    for got, ref in ((dq, qr.grad), (dk, kr.grad), (dv, vr.grad)):
        assert np.abs(got - ref.numpy()).max() < 1e-12


def test_backward_finite_differences_tiny():
    """Central differences of sum(O * dO) on a 1 x 1 x 3 x 2 problem."""
    g = np.random.default_rng(12)
    q, k, v, do = (g.standard_normal((1, 1, 3, 2)) for _ in range(4))
    dq, dk, dv = A.attention_backward(q, k, v, do, True, 0.7)
    f = lambda qq, kk, vv: float((A.attention(qq, kk, vv, True, 0.7)[0] * do).sum())
    eps = 1e-6
    for arr, grad, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += eps
            args_m[which][idx] -= eps
            num[idx] = (f(*args_p) - f(*args_m)) / (2 * eps)
        assert np.abs(num - grad).max() < 1e-7


def test_backward_row_statistic_identity():
    """sum_k P_ik dP_ik = sum_c dO_ic O_ic, the per-row quantity the tiled
    backward computes from the stored O instead of from P."""
    g = torch.Generator().manual_seed(2)
    q, k, v, do = (torch.randn(1, 1, 6, 4, generator=g, dtype=torch.float64) for _ in range(4))
    O, _ = A.attention(q, k, v, False, 0.5)
    P = A.softmax_rows(q, k, False, 0.5)
    dP = do.numpy() @ v.numpy().transpose(0, 1, 3, 2)
    assert np.abs((P * dP).sum(-1) - (do.numpy() * O).sum(-1)).max() < 1e-12


def _packed_mask(cu_q, cu_k, causal):
    """Boolean [total_q][total_k]: query row i sees key j iff both belong to the
    same sequence (and, causal, j - k0 <= (i - q0) + (nk - nq))."""
    tq, tk = cu_q[-1], cu_k[-1]
    m = torch.zeros(tq, tk, dtype=torch.bool)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        i = torch.arange(q0, q1)[:, None] - q0
        j = torch.arange(k0, k1)[None, :] - k0
        vis = torch.ones(q1 - q0, k1 - k0, dtype=torch.bool)
        if causal:
            vis = j <= i + ((k1 - k0) - (q1 - q0))
        m[q0:q1, k0:k1] = vis
    return m


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2)])
def test_varlen_matches_block_diagonal_sdpa(causal, Hq, Hkv):
    """The packed batch equals one attention over the concatenation with a
    block-diagonal mask (PyTorch SDPA, fp64), and LSE equals the masked
    log-sum-exp; rows that see no key (empty key set, or causal with fewer
    keys than queries) get O = 0, LSE = -inf."""
    lq = [5, 0, 17, 3, 9]
    lk = [7, 4, 17, 0, 4]
    cu_q = np.concatenate([[0], np.cumsum(lq)])
    cu_k = np.concatenate([[0], np.cumsum(lk)])
    g = torch.Generator().manual_seed(11)
    d = 8
    q = torch.randn(cu_q[-1], Hq, d, generator=g, dtype=torch.float64)
    k = torch.randn(cu_k[-1], Hkv, d, generator=g, dtype=torch.float64)
    v = torch.randn(cu_k[-1], Hkv, d, generator=g, dtype=torch.float64)
    O, L = A.attention_varlen(q, k, v, cu_q, cu_k, causal, 0.3)
    mask = _packed_mask(cu_q, cu_k, causal)
    rep = Hq // Hkv
    kh, vh = k.repeat_interleave(rep, dim=1), v.repeat_interleave(rep, dim=1)
    s = torch.einsum("ihd,jhd->hij", q, kh) * 0.3
    s = s.masked_fill(~mask[None], float("-inf"))
    lse = torch.logsumexp(s, dim=-1)                        # [H][total_q]
    seen = mask.any(dim=1).numpy()
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(0, 1)[None], kh.transpose(0, 1)[None], vh.transpose(0, 1)[None],
        attn_mask=mask[None, None], scale=0.3)[0].transpose(0, 1).numpy()
    np.testing.assert_allclose(O[seen], ref[seen], rtol=0, atol=1e-12)
    assert (O[~seen] == 0).all() and np.isneginf(L[:, ~seen]).all()
    np.testing.assert_allclose(L[:, seen], lse.numpy()[:, seen], rtol=0, atol=1e-12)
    assert (~seen).sum() > 0                                 # the case is covered


def test_decode_varlen_matches_masked_sdpa():
    B, Hq, Hkv, N, d = 4, 4, 2, 23, 8
    lens = [23, 0, 1, 11]
    g = torch.Generator().manual_seed(12)
    q = torch.randn(B, Hq, 1, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64)
    O, L = A.decode_varlen(q, k, v, lens, 0.5)
    keep = torch.arange(N)[None, :] < torch.tensor(lens)[:, None]          # [B][N]
    kh, vh = k.repeat_interleave(2, dim=1), v.repeat_interleave(2, dim=1)
    for b in range(B):
        if lens[b] == 0:
            assert (O[b] == 0).all() and np.isneginf(L[b]).all()
            continue
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[b:b + 1], kh[b:b + 1], vh[b:b + 1], attn_mask=keep[b][None, None, None], scale=0.5)
        np.testing.assert_allclose(O[b], ref[0].numpy(), rtol=0, atol=1e-12)
        s = (q[b] @ kh[b].transpose(-1, -2) * 0.5)[..., : lens[b]]
        np.testing.assert_allclose(L[b], torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-12)


def test_backward_fp8_p_closed_form():
    """Keys with identical scores give P = 1/n on every visible key.  For
    n = 2, 4 the value is an e4m3 value and rounding changes nothing; for
    n = 3, e4m3(1/3) = 0.34375 (the nearer of 0.3125 and 0.34375), so
    dV_j = 0.34375 * sum of dO over the rows that see key j, while dQ and
    dK are those of the unrounded backward."""
    from oracle import fp8 as F
    g = np.random.default_rng(21)
    d = 4
    for n, p8 in ((2, 0.5), (4, 0.25), (3, 0.34375)):
        q = g.standard_normal((1, 1, 5, d))
        k = np.tile(g.standard_normal(d), (n, 1))[None, None]      # identical keys
        v = g.standard_normal((1, 1, n, d))
        do = g.standard_normal((1, 1, 5, d))
        dq0, dk0, dv0 = A.attention_backward(q, k, v, do, False, 0.7)
        dq8, dk8, dv8 = A.attention_backward(q, k, v, do, False, 0.7, p_round=F.e4m3_encode_value)
        np.testing.assert_allclose(dv8[0, 0], np.tile(p8 * do[0, 0].sum(axis=0), (n, 1)), rtol=0, atol=1e-12)
        np.testing.assert_array_equal(dq8, dq0)
        np.testing.assert_array_equal(dk8, dk0)
        if n != 3:
            np.testing.assert_allclose(dv8, dv0, rtol=0, atol=1e-12)
