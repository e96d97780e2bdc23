"""Property-based pins of the oracle (hypothesis, CPU): invariants that must
hold for every shape, not only the hand-picked cases of the other oracle
tests.  Sizes stay small so the whole file runs in seconds."""
import math

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import attention as A
from oracle import fp8 as F
from oracle import lowp as L

SETTINGS = settings(max_examples=25, deadline=None, suppress_health_check=[HealthCheck.too_slow])


def _qkv(seed, B, H, Nq, Nkv, d, scale=1.0):
    g = np.random.default_rng(seed)
    return (g.standard_normal((B, H, Nq, d)) * scale, g.standard_normal((B, H, Nkv, d)) * scale,
            g.standard_normal((B, H, Nkv, d)))


@SETTINGS
@given(seed=st.integers(0, 10_000), Nq=st.integers(1, 40), Nkv=st.integers(1, 40), d=st.sampled_from([4, 8]),
       Br=st.sampled_from([1, 3, 8, 16]), Bc=st.sampled_from([1, 5, 8, 16]), causal=st.booleans())
def test_pages_blockwise_algorithm_equals_definition(seed, Nq, Nkv, d, Br, Bc, causal):
    """The tiled algorithm (any block sizes, ragged tails) reproduces the
    definition, including rows that see no key."""
    q, k, v = _qkv(seed, 1, 2, Nq, Nkv, d)
    O, L_ = A.attention(q, k, v, causal, 0.7)
    Ob, Lb = A.attention_blockwise(q, k, v, causal, 0.7, Br, Bc)
    np.testing.assert_allclose(Ob, O, rtol=1e-11, atol=1e-11)
    fin = np.isfinite(L_)
    assert np.array_equal(np.isfinite(Lb), fin)
    np.testing.assert_allclose(Lb[fin], L_[fin], rtol=1e-11, atol=1e-11)


@SETTINGS
@given(seed=st.integers(0, 10_000), Nq=st.integers(1, 30), Nkv=st.integers(1, 30),
       Bc=st.sampled_from([1, 4, 7, 16]), tau=st.sampled_from([0.0, 2.0, 8.0]), causal=st.booleans(),
       spread=st.sampled_from([1.0, 10.0]))
def test_lazy_rescale_equals_definition(seed, Nq, Nkv, Bc, tau, causal, spread):
    q, k, v = _qkv(seed, 1, 1, Nq, Nkv, 8, spread)
    O, L_ = A.attention(q, k, v, causal, 0.5)
    Ol, Ll = A.attention_lazy_rescale(q, k, v, causal, 0.5, Bc, tau)
    np.testing.assert_allclose(Ol, O, rtol=1e-10, atol=1e-10)
    fin = np.isfinite(L_)
    np.testing.assert_allclose(Ll[fin], L_[fin], rtol=1e-10, atol=1e-10)


@SETTINGS
@given(seed=st.integers(0, 10_000), Nkv=st.integers(1, 60), splits=st.integers(1, 70))
def test_split_kv_combine_equals_unsplit(seed, Nkv, splits):
    q, k, v = _qkv(seed, 2, 2, 1, Nkv, 8)
    O, L_ = A.decode(q, k, v, 0.3)
    Oc, Lc = A.combine(*A.decode_partials(q, k, v, 0.3, splits))
    np.testing.assert_allclose(Oc, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lc, L_, rtol=0, atol=1e-12)


@SETTINGS
@given(seed=st.integers(0, 10_000), lens=st.lists(st.tuples(st.integers(0, 12), st.integers(0, 12)),
                                                   min_size=1, max_size=5), causal=st.booleans())
def test_varlen_equals_each_sequence_alone(seed, lens, causal):
    lq = [a for a, _ in lens]
    lk = [b for _, b in lens]
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int64)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int64)
    g = np.random.default_rng(seed)
    q = g.standard_normal((cu_q[-1], 2, 4))
    k = g.standard_normal((cu_k[-1], 1, 4))
    v = g.standard_normal((cu_k[-1], 1, 4))
    O, L_ = A.attention_varlen(q, k, v, cu_q, cu_k, causal, 0.9)
    for b in range(len(lens)):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        if q1 == q0:
            continue
        if k1 == k0:
            assert (O[q0:q1] == 0).all() and np.isneginf(L_[:, q0:q1]).all()
            continue
        Ob, Lb = A.attention_gqa(q[q0:q1].transpose(1, 0, 2)[None], k[k0:k1].transpose(1, 0, 2)[None],
                                 v[k0:k1].transpose(1, 0, 2)[None], causal, 0.9)
        np.testing.assert_allclose(O[q0:q1], Ob[0].transpose(1, 0, 2), rtol=0, atol=1e-13)


@SETTINGS
@given(seed=st.integers(0, 10_000), rows=st.integers(1, 20), scale=st.sampled_from([1e-3, 1.0, 30.0]))
def test_int8_and_int4_row_quantisers_round_to_within_half_a_step(seed, rows, scale):
    x = np.random.default_rng(seed).standard_normal((rows, 16)).astype(np.float32) * scale
    for quant, qmax in ((L.quantize_int8_rows, 127), (L.quantize_int4_rows, 7)):
        q, s = quant(x)
        assert np.abs(q).max() <= qmax
        assert (np.abs(x.astype(np.float64) - q * s[:, None].astype(np.float64))
                <= s[:, None].astype(np.float64) * (0.5 + 1e-6)).all()


@SETTINGS
@given(seed=st.integers(0, 10_000), rows=st.integers(1, 12), rotate=st.booleans(),
       outlier=st.sampled_from([1.0, 50.0]))
def test_fp8_row_quantiser_error_within_half_an_e4m3_step(seed, rows, rotate, outlier):
    """Every code is within half an e4m3 step of y / s (the rotated row when
    rotating), the row max maps to +-448, and H_d^T applied to the rotated
    row recovers d times the (signed) input."""
    g = np.random.default_rng(seed)
    x = g.standard_normal((rows, 64)).astype(np.float32)
    x[:, 3] *= outlier
    signs = np.where(g.random(64) < 0.5, -1.0, 1.0) if rotate else None
    qv, s = F.quantize_fp8_rows(x, signs)
    y = F.fwht_f32(x * signs.astype(np.float32)) if rotate else x
    t = y.astype(np.float64) / s[:, None].astype(np.float64)
    a = np.abs(t)
    # spacing of e4m3 around |t|: 2^(e - 3) in the normal range, 2^-9 below 2^-6
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    step = 2.0 ** (e - 3)
    assert (np.abs(qv - t) <= step / 2 * (1 + 1e-6)).all()
    assert np.allclose(np.abs(qv).max(axis=1), 448.0)
    if rotate:
        back = F.fwht_f32(y) / 64.0 * signs
        np.testing.assert_allclose(back, x, rtol=1e-5, atol=1e-5 * outlier)


@SETTINGS
@given(seed=st.integers(0, 10_000), Nq=st.integers(1, 20), Nkv=st.integers(1, 20), causal=st.booleans())
def test_backward_gradient_of_sum_of_o_times_dout_is_consistent(seed, Nq, Nkv, causal):
    """Directional derivative: for a random direction (dq, dk, dv), the change
    of <O, dO> to first order equals <grad, direction> (central differences)."""
    q, k, v = _qkv(seed, 1, 1, Nq, Nkv, 4)
    do = np.random.default_rng(seed + 1).standard_normal(q.shape)
    gq, gk, gv = A.attention_backward(q, k, v, do, causal, 0.8)
    g = np.random.default_rng(seed + 2)
    uq, uk, uv = g.standard_normal(q.shape), g.standard_normal(k.shape), g.standard_normal(v.shape)
    h = 1e-5

    def f(t):
        O, _ = A.attention(q + t * uq, k + t * uk, v + t * uv, causal, 0.8)
        return float((O * do).sum())
    num = (f(h) - f(-h)) / (2 * h)
    ana = float((gq * uq).sum() + (gk * uk).sum() + (gv * uv).sum())
    assert math.isclose(num, ana, rel_tol=1e-5, abs_tol=1e-6)
