"""Pins of the boundary-flip handling of the quantised oracles (CPU only).

* ``ratio_range`` (the exact extremes of a ratio of linear functions over a
  finite product of choices) against brute-force enumeration;
* ``near_midpoint``: a value one fp32 ulp either side of a rounding midpoint
  of the INT8, e2m1 or e4m3 grid is flagged and gets the other neighbour; a
  value far from every midpoint is not flagged;
* end to end, for each quantised forward: inputs built so that one element
  (or, for quantise-after-exp, one block scale) sits on a rounding midpoint.
  The element is flagged, and the two outcomes are REALISED by nudging the
  input a hair to either side and re-running the oracle; the interval of the
  unnudged run must be exactly the hull of those two results.  Rows with
  nothing flagged get an interval of width exactly zero.
"""
import itertools

import numpy as np
import pytest

from oracle import attention as A
from oracle import fp8 as F
from oracle import lowp as Q
from oracle.outcomes import eval_band, near_midpoint, ratio_range

LN2 = float(np.log(2.0))


# ------------------------------------------------------------ ratio_range
def _brute(num, den, opt_a, opt_b):
    V, K, d = opt_a.shape
    vals = []
    for choice in itertools.product(range(K + 1), repeat=V):
        a = num.copy()
        b = den
        for v, k in enumerate(choice):
            if k:
                a = a + opt_a[v, k - 1]
                b = b + opt_b[v, k - 1]
        vals.append(a / b)
    vals = np.array(vals)
    return vals.min(axis=0), vals.max(axis=0)


@pytest.mark.parametrize("seed", range(12))
def test_ratio_range_equals_brute_force(seed):
    rng = np.random.default_rng(seed)
    V = int(rng.integers(1, 6))
    K = int(rng.integers(1, 4))
    d = 5
    num = rng.normal(size=d) * 3
    den = 1.0 + rng.random()
    opt_a = rng.normal(size=(V, K, d))
    opt_b = rng.normal(size=(V, K)) * 0.1           # both signs
    lo, hi = ratio_range(num, den, opt_a, opt_b)
    blo, bhi = _brute(num, den, opt_a, opt_b)
    np.testing.assert_allclose(lo, blo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(hi, bhi, rtol=0, atol=1e-12)


def test_ratio_range_without_variables_is_the_point():
    num = np.array([1.0, -2.0, 3.0])
    lo, hi = ratio_range(num, 2.0, np.zeros((0, 1, 3)), np.zeros((0, 1)))
    assert np.array_equal(lo, num / 2.0) and np.array_equal(hi, num / 2.0)


def test_ratio_range_refuses_a_non_positive_row_sum():
    with pytest.raises(ValueError):
        ratio_range(np.ones(2), 1.0, np.zeros((1, 1, 2)), np.array([[-1.5]]))


# ------------------------------------------------------------ near_midpoint
def _ulps(v):
    v32 = np.float32(v)
    return [float(np.nextafter(v32, np.float32(-np.inf))), float(np.nextafter(v32, np.float32(np.inf)))]


E4M3 = Q.UE4M3_VALUES
GRIDS = {
    "int8": np.arange(128.0),
    "e2m1": Q.E2M1_VALUES,
    "e4m3": E4M3,
}


@pytest.mark.parametrize("grid", list(GRIDS))
def test_one_ulp_from_a_midpoint_is_flagged(grid):
    g = GRIDS[grid]
    mids = (g[1:] + g[:-1]) / 2.0
    for i in range(0, mids.size, max(1, mids.size // 17)):
        t = mids[i]
        for y in _ulps(t):
            base = g[i] if y < t else g[i + 1]
            band = eval_band(y, 0.5, 0.0, 0.0)          # the model's band at |x| + |m| = 1/2
            flag, alt = near_midpoint(np.array([y]), g, np.array([base]), band)
            assert flag[0], (grid, t, y)
            assert alt[0] == (g[i + 1] if base == g[i] else g[i])


@pytest.mark.parametrize("grid", list(GRIDS))
def test_far_from_every_midpoint_is_not_flagged(grid):
    g = GRIDS[grid]
    y = g[1:-1]                                        # grid values themselves
    band = eval_band(y, 3.0, 5.0, 1e-7)
    flag, alt = near_midpoint(y, g, y, band)
    assert not flag.any()
    assert np.array_equal(alt, y)
    # a quarter of the way between two neighbours is far away as well
    q = g[1:-1] + (g[2:] - g[1:-1]) / 4
    flag, _ = near_midpoint(q, g, g[1:-1], eval_band(q, 3.0, 5.0, 1e-7))
    assert not flag.any()


def test_band_model():
    assert eval_band(0.0, 10.0, 10.0, 1e-4) == 1e-4
    b = eval_band(100.0, 2.0, 3.0, 0.0)
    assert b == pytest.approx(100.0 * (LN2 * 2e-6 * 6.0 + 2.0 ** -20))


# ------------------------------------------------------------ INT8 end to end
def _int8_case(ks1, d=16):
    """One query row, keys 0..3: x_0 = 0 (the row max), x_1 = -ks1 (scale =
    ln 2, s_Q = 1, so x = S * s_K), x_2 = -2.3, x_3 = -0.37; V codes random."""
    qi = np.zeros((1, 1, 1, d), np.int8)
    qi[..., 0] = 1
    ki = np.zeros((1, 1, 4, d), np.int8)
    ki[0, 0, 1, 0] = -1
    ki[0, 0, 2, 0] = -1
    ki[0, 0, 3, 0] = -1
    qs = np.ones((1, 1, 1), np.float32)
    ks = np.array([[[1.0, ks1, 2.3, 0.37]]], np.float32)
    vi = np.random.default_rng(0).integers(-127, 128, size=(1, 1, 4, d)).astype(np.int8)
    vs = np.array([[0.05]], np.float32)
    return qi, qs, ki, ks, vi, vs


def test_int8_midpoint_is_flagged_and_both_outcomes_lie_in_the_interval():
    # 127 * 2^-1 = 63.5: the tie between P8 = 63 and 64
    qi, qs, ki, ks, vi, vs = _int8_case(1.0)
    O, L, R = Q.attention_int8(qi, qs, ki, ks, vi, vs, scale=LN2, outcomes=True)
    assert R.flips == 1 and R.flagged_rows == 1
    outs = []
    for nudge in (1 - 1e-6, 1 + 1e-6):
        args = _int8_case(nudge)
        Oa, La = Q.attention_int8(*args, scale=LN2)
        outs.append((Oa, La))
    Os = np.stack([o for o, _ in outs])
    Ls = np.stack([lse for _, lse in outs])
    assert not np.array_equal(Os[0], Os[1])              # the two roundings differ
    np.testing.assert_allclose(R.O_lo, Os.min(axis=0), rtol=0, atol=1e-12)
    np.testing.assert_allclose(R.O_hi, Os.max(axis=0), rtol=0, atol=1e-12)
    np.testing.assert_allclose(R.LSE_lo, Ls.min(axis=0), rtol=0, atol=1e-12)
    np.testing.assert_allclose(R.LSE_hi, Ls.max(axis=0), rtol=0, atol=1e-12)
    assert R.distance(O, L) == (0.0, 0.0)


def test_int8_nothing_flagged_gives_width_zero():
    qi, qs, ki, ks, vi, vs = _int8_case(0.77)            # 127 * 2^-0.77 = 74.6: no midpoint near
    O, L, R = Q.attention_int8(qi, qs, ki, ks, vi, vs, scale=LN2, outcomes=True)
    assert R.flips == 0 and R.flagged_rows == 0 and R.width() == 0.0
    assert np.array_equal(R.O_lo, O) and np.array_equal(R.O_hi, O)
    assert np.array_equal(R.LSE_lo, L) and np.array_equal(R.LSE_hi, L)


def test_int8_unflagged_rows_keep_the_plain_value_on_random_inputs():
    rng = np.random.default_rng(5)
    qi = rng.integers(-127, 128, size=(1, 2, 40, 32)).astype(np.int8)
    ki = rng.integers(-127, 128, size=(1, 2, 300, 32)).astype(np.int8)
    vi = rng.integers(-127, 128, size=(1, 2, 300, 32)).astype(np.int8)
    qs = rng.uniform(0.001, 0.01, size=(1, 2, 40)).astype(np.float32)
    ks = rng.uniform(0.001, 0.01, size=(1, 2, 300)).astype(np.float32)
    vs = np.array([[0.02, 0.03]], np.float32)
    O, L, R = Q.attention_int8(qi, qs, ki, ks, vi, vs, causal=True, outcomes=True)
    flagged = R.O_hi != R.O_lo
    rows_changed = flagged.any(axis=-1)
    assert rows_changed.sum() <= R.flagged_rows
    assert np.array_equal(R.O_lo[~rows_changed], O[~rows_changed])
    assert (R.O_lo <= O + 1e-15).all() and (O <= R.O_hi + 1e-15).all()


# ------------------------------------------------------------ FP4 end to end
def _fp4_case(c1, d=16, nk=32):
    """Dequantised operands with x = q . k * ln2 * log2(e): key 0 at x = 0,
    key 1 at x = c1, the rest spread below."""
    q = np.zeros((1, 1, 1, d))
    q[..., 0] = 1.0
    k = np.zeros((1, 1, nk, d))
    k[0, 0, 1, 0] = c1
    k[0, 0, 2:, 0] = -np.linspace(0.3, 6.0, nk - 2)
    v = np.random.default_rng(1).normal(size=(1, 1, nk, d))
    return q, k, v


def test_fp4_direct_p_midpoint_flagged_and_both_outcomes_realised():
    c = float(np.log2(3.5 / 6.0))                         # 6 * 2^c = 3.5, midpoint of 3 and 4
    q, k, v = _fp4_case(c)
    O, L, R = Q.attention_fp4(q, k, v, Q.DIRECT_P, scale=LN2, outcomes=True)
    assert R.flips >= 1
    Os = np.stack([Q.attention_fp4(*_fp4_case(c + s), Q.DIRECT_P, scale=LN2)[0] for s in (-1e-6, 1e-6)])
    assert not np.array_equal(Os[0], Os[1])
    assert (R.O_lo <= Os.min(axis=0) + 1e-12).all() and (Os.max(axis=0) <= R.O_hi + 1e-12).all()
    if R.flips == 1:
        np.testing.assert_allclose(R.O_lo, Os.min(axis=0), atol=1e-12)
        np.testing.assert_allclose(R.O_hi, Os.max(axis=0), atol=1e-12)


def test_fp4_quant_after_exp_scale_midpoint_flips_the_block():
    """Keys 16..31 form one 16-key scale block whose amax is p_16 =
    2^(x_16); amax / 6 = 0.08203125 is the midpoint of the e4m3 values
    0.078125 and 0.0859375, so the block scale (and with it the block's codes)
    may take either value.  Both are realised by nudging x_16."""
    d, nk = 16, 32
    amax = 6.0 * (0.078125 + 0.0859375) / 2.0
    q = np.zeros((1, 1, 1, d))
    q[..., 0] = 1.0

    def make(x16):
        k = np.zeros((1, 1, nk, d))
        k[0, 0, 1:16, 0] = -np.linspace(0.5, 3.0, 15)
        k[0, 0, 16, 0] = x16
        k[0, 0, 17:, 0] = np.log2(np.linspace(0.05, 0.45, nk - 17))
        return k

    v = np.random.default_rng(2).normal(size=(1, 1, nk, d))
    x16 = float(np.log2(amax))
    O, L, R = Q.attention_fp4(q, make(x16), v, Q.QUANT_AFTER_EXP, scale=LN2, outcomes=True)
    assert R.flips >= 1
    Os = np.stack([Q.attention_fp4(q, make(x16 + s), v, Q.QUANT_AFTER_EXP, scale=LN2)[0]
                   for s in (-1e-5, 1e-5)])
    assert not np.array_equal(Os[0], Os[1])                # the two scales give different codes
    assert (R.O_lo <= Os.min(axis=0) + 1e-9).all() and (Os.max(axis=0) <= R.O_hi + 1e-9).all()


def test_fp4_random_rows_contain_the_oracle_value_and_unflagged_rows_are_points():
    rng = np.random.default_rng(7)
    q = rng.normal(size=(1, 1, 64, 32)) * 2
    k = rng.normal(size=(1, 1, 200, 32)) * 2
    v = rng.normal(size=(1, 1, 200, 32))
    for mode in (Q.DIRECT_P, Q.QUANT_AFTER_EXP):
        O, L, R = Q.attention_fp4(q, k, v, mode, outcomes=True)
        assert (R.O_lo <= O + 1e-15).all() and (O <= R.O_hi + 1e-15).all()
        assert R.flagged_rows <= R.rows
        point = (R.O_hi == R.O_lo).all(axis=-1)
        assert point.sum() >= R.rows - R.flagged_rows


# ------------------------------------------------------------ FP8 end to end
def _fp8_case(ks1, d=16):
    qv = np.zeros((1, 1, 1, d))
    qv[..., 0] = 1.0
    kv = np.zeros((1, 1, 3, d))
    kv[0, 0, 1, 0] = -1.0
    kv[0, 0, 2, 0] = -1.0
    qs = np.ones((1, 1, 1), np.float32)
    ks = np.array([[[1.0, ks1, 3.1]]], np.float32)
    vv = F.e4m3_encode_value(np.random.default_rng(3).normal(size=(1, 1, 3, d)) * 50)
    vs = np.full((1, 1, d), 0.01, np.float32)
    return qv, qs, kv, ks, vv, vs


def test_fp8_midpoint_flagged_and_both_outcomes_realised():
    t = (0.5 + 0.5625) / 2.0                              # e4m3 midpoint
    c = float(-np.log2(t))
    O, L, R = F.attention_fp8(*_fp8_case(c), scale=LN2, outcomes=True)
    assert R.flips == 1 and R.ambiguous_rescales == 0
    Os = np.stack([F.attention_fp8(*_fp8_case(c * f), scale=LN2)[0] for f in (1 - 1e-5, 1 + 1e-5)])
    assert not np.array_equal(Os[0], Os[1])
    np.testing.assert_allclose(R.O_lo, Os.min(axis=0), atol=1e-12)
    np.testing.assert_allclose(R.O_hi, Os.max(axis=0), atol=1e-12)


def test_fp8_rescale_decision_on_the_threshold_is_reported():
    """Two 128-key blocks: the second block's max exceeds the first's by
    exactly tau = 8, so a device may or may not move its reference."""
    d = 16
    qv = np.zeros((1, 1, 1, d))
    qv[..., 0] = 1.0
    kv = np.zeros((1, 1, 256, d))
    kv[0, 0, :128, 0] = -np.linspace(0.0, 1.0, 128)
    kv[0, 0, 128:, 0] = 8.0 - np.linspace(0.0, 1.0, 128)
    qs = np.ones((1, 1, 1), np.float32)
    ks = np.ones((1, 1, 256), np.float32)
    vv = np.ones((1, 1, 256, d))
    vs = np.ones((1, 1, d), np.float32)
    *_, R = F.attention_fp8(qv, qs, kv, ks, vv, vs, scale=LN2, outcomes=True, tau=8.0)
    assert R.ambiguous_rescales == 1
    *_, R = F.attention_fp8(qv, qs, kv * 0.9, ks, vv, vs, scale=LN2, outcomes=True, tau=8.0)
    assert R.ambiguous_rescales == 0


def test_fp8_both_rescale_decisions_lie_in_the_hull():
    """As above with values that make the two decisions give different
    outputs.  On the threshold the two references differ by exactly 2^8, and
    e4m3 rounding commutes with powers of two except in its subnormal range,
    so the second block's scores spread down to 19 below its max (subnormal
    under one reference, normal under the other).  Nudging that block's max
    below / above the threshold realises each decision."""
    d = 16
    rng = np.random.default_rng(4)
    qv = np.zeros((1, 1, 1, d))
    qv[..., 0] = 1.0
    qs = np.ones((1, 1, 1), np.float32)
    ks = np.ones((1, 1, 256), np.float32)
    vv = F.e4m3_encode_value(rng.normal(size=(1, 1, 256, d)) * 30)
    vs = np.full((1, 1, d), 0.02, np.float32)

    def keys(top):
        kv = np.zeros((1, 1, 256, d))
        kv[0, 0, :128, 0] = -rng.uniform(0.0, 3.0, 128)
        kv[0, 0, 0, 0] = 0.0
        kv[0, 0, 128:, 0] = top - np.linspace(0.0, 19.0, 128) ** 1.01
        return kv

    base = keys(8.0)
    O, L, R = F.attention_fp8(qv, qs, base, ks, vv, vs, scale=LN2, outcomes=True, tau=8.0)
    assert R.ambiguous_rescales == 1
    outs = []
    for s in (-4e-6, 4e-6):                              # a few fp32 ulps of 8 (S is rounded to fp32)
        kv = base.copy()
        kv[0, 0, 128:, 0] += s
        outs.append(F.attention_fp8(qv, qs, kv, ks, vv, vs, scale=LN2, tau=8.0))
    Os = np.stack([o for o, _ in outs])
    Ls = np.stack([lse for _, lse in outs])
    assert np.abs(Os[0] - Os[1]).max() > 1e-4            # the decisions give different outputs
    # the nudge itself moves O and LSE continuously by ~ln2 * 4e-6 relative
    tol = 1e-5
    assert (R.O_lo <= Os.min(axis=0) + tol).all() and (Os.max(axis=0) <= R.O_hi + tol).all()
    assert (R.LSE_lo <= Ls.min(axis=0) + tol).all() and (Ls.max(axis=0) <= R.LSE_hi + tol).all()


# ------------------------------------------------------------ FP8-P backward
def test_backward_fp8p_dv_interval_equals_brute_force():
    """dV = round(P)^T dO is linear in the rounded P: with a wide flag band
    (so that several elements are flagged) the interval must equal the range
    over every combination of roundings."""
    rng = np.random.default_rng(11)
    q, k, v, do = (rng.normal(size=(1, 1, n, 4)) for n in (2, 3, 3, 2))
    grid = E4M3
    _, _, dv, (lo, hi) = A.attention_backward(q, k, v, do, p_round=F.e4m3_encode_value, p_grid=grid, p_rel=0.08)
    P = A.softmax_rows(q, k)[0, 0]
    base = F.e4m3_encode_value(P)
    flag, alt = near_midpoint(P, grid, base, 0.08 * P)
    idx = np.argwhere(flag)
    assert 1 <= len(idx) <= 6
    vals = []
    for choice in itertools.product((0, 1), repeat=len(idx)):
        Pc = base.copy()
        for (i, j), c in zip(idx, choice):
            if c:
                Pc[i, j] = alt[i, j]
        vals.append(Pc.T @ do[0, 0])
    vals = np.array(vals)
    np.testing.assert_allclose(lo[0, 0], vals.min(axis=0), atol=1e-14)
    np.testing.assert_allclose(hi[0, 0], vals.max(axis=0), atol=1e-14)
    np.testing.assert_allclose(dv[0, 0], base.T @ do[0, 0], atol=1e-14)


def test_a_planted_error_outside_the_interval_fails_the_check():
    """The GPU tests' check (tests._parity.assert_within_outcomes) accepts
    either realised rounding and rejects an output moved 2x the tolerance
    beyond the interval."""
    from tests._parity import Q_O_ABS, assert_within_outcomes
    import torch
    qi, qs, ki, ks, vi, vs = _int8_case(1.0)
    O, L, R = Q.attention_int8(qi, qs, ki, ks, vi, vs, scale=LN2, outcomes=True)
    n = 10_000  # the case is built to sit on a midpoint: keep the flag-rate check out of it
    for nudge in (1 - 1e-6, 1 + 1e-6):
        Oa, La = Q.attention_int8(*_int8_case(nudge), scale=LN2)
        assert_within_outcomes(torch.from_numpy(Oa), torch.from_numpy(La), O, L, R, "realised", n)
    bad = R.O_hi + 2 * Q_O_ABS
    with pytest.raises(AssertionError):
        assert_within_outcomes(torch.from_numpy(bad), torch.from_numpy(L), O, L, R, "planted", n)
