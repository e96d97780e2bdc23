"""Pins of the INT8 / FP4 parts of the oracle: format tables from the OCP
specifications (tests/golden), exhaustive encoder properties, inputs on which
quantisation is the identity, brute force on tiny inputs, and the bound that
the quantised forwards keep to the exact fp64 attention.  No GPU."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import lowp as Q

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(7)


def _table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                c, v = line.split()
                rows.append((int(c, 0), float(v)))
    return rows


# ---------------------------------------------------------------- INT8 ------

def test_int8_rows_identity_on_integer_rows_with_amax_127():
    x = RNG.integers(-127, 128, size=(3, 5, 64)).astype(np.float64)
    x[..., 3] = 127.0
    q, s = Q.quantize_int8_rows(x)
    assert (s == 1.0).all() and np.array_equal(q.astype(np.float64), x)


def test_int8_rows_zero_row_and_known_values():
    x = np.array([[0.0, 0.0, 0.0, 0.0], [2.0, -1.0, 0.5, 1.0]])
    q, s = Q.quantize_int8_rows(x)
    assert s[0] == 1.0 and (q[0] == 0).all()
    # s = 2/127; 1/s = 63.5 exactly in real arithmetic, so the fp32 quotient
    # sits at a tie or one ulp off it -> 63 or 64 depending on rounding of s.
    assert q[1, 0] == 127 and q[1, 1] in (-63, -64) and q[1, 3] in (63, 64)
    assert s.dtype == np.float32 and s[1] == np.float32(np.float32(2.0) / np.float32(127.0))


def test_int8_quantise_error_bound():
    x = RNG.standard_normal((4, 128)) * 3
    q, s = Q.quantize_int8_rows(x)
    err = np.abs(q * s[:, None].astype(np.float64) - x)
    assert (err <= s[:, None] * (0.5 + 1e-5)).all()
    assert (np.abs(q) <= 127).all()


def test_int8_heads_one_scale_per_head():
    x = RNG.standard_normal((2, 3, 10, 8))
    q, s = Q.quantize_int8_heads(x)
    assert s.shape == (2, 3)
    np.testing.assert_allclose(s, np.abs(x).max(axis=(2, 3)) / 127, rtol=1e-6)
    assert np.abs(q).max() == 127


def test_int8_scores_brute_force():
    qi = RNG.integers(-127, 128, size=(1, 1, 3, 5)).astype(np.int8)
    ki = RNG.integers(-127, 128, size=(1, 1, 4, 5)).astype(np.int8)
    S = Q.int8_scores(qi, ki)
    for i in range(3):
        for j in range(4):
            assert S[0, 0, i, j] == sum(int(qi[0, 0, i, c]) * int(ki[0, 0, j, c]) for c in range(5))


def _int8_brute(qi, qs, ki, ks, vi, vs, scale, Bc, causal):
    """Pure-Python loops over one (b, h): the INT8 steps in order."""
    Nq, d = qi.shape
    Nkv = ki.shape[0]
    O = np.zeros((Nq, d))
    L = np.zeros(Nq)
    for i in range(Nq):
        m, l, acc = -math.inf, 0.0, [0.0] * d
        for j0 in range(0, Nkv, Bc):
            xs = []
            for j in range(j0, min(Nkv, j0 + Bc)):
                if causal and j > i + Nkv - Nq:
                    xs.append((j, -math.inf))
                    continue
                s = sum(int(qi[i, c]) * int(ki[j, c]) for c in range(d))
                xs.append((j, s * float(qs[i]) * float(ks[j]) * scale / math.log(2)))
            mb = max(x for _, x in xs)
            if mb > m:
                f = 0.0 if m == -math.inf else 2.0 ** (m - mb)
                acc = [a * f for a in acc]
                l *= f
                m = mb
            for j, x in xs:
                if x == -math.inf:
                    continue
                p8 = float(np.rint(127.0 * 2.0 ** (x - m)))
                l += p8 / 127.0
                for c in range(d):
                    acc[c] += p8 * int(vi[j, c]) * float(vs) / 127.0
        O[i] = [a / l for a in acc]
        L[i] = math.log(2) * (m + math.log2(l))
    return O, L


@pytest.mark.parametrize("causal", [False, True])
def test_int8_emulation_brute_force(causal):
    x = RNG.standard_normal((1, 1, 5, 4)) * 2
    y = RNG.standard_normal((1, 1, 7, 4)) * 2
    z = RNG.standard_normal((1, 1, 7, 4))
    qi, qs = Q.quantize_int8_rows(x)
    ki, ks = Q.quantize_int8_rows(y)
    vi, vs = Q.quantize_int8_heads(z)
    O, L = Q.attention_int8(qi, qs, ki, ks, vi, vs, causal, 0.7, Bc=3)
    Ob, Lb = _int8_brute(qi[0, 0], qs[0, 0], ki[0, 0], ks[0, 0], vi[0, 0], vs[0, 0], 0.7, 3, causal)
    np.testing.assert_allclose(O[0, 0], Ob, atol=1e-12)
    np.testing.assert_allclose(L[0, 0], Lb, atol=1e-12)


def test_int8_emulation_close_to_exact_attention():
    x, y, z = (RNG.standard_normal((1, 2, n, 64)) for n in (40, 300, 300))
    qi, qs = Q.quantize_int8_rows(x)
    ki, ks = Q.quantize_int8_rows(y)
    vi, vs = Q.quantize_int8_heads(z)
    O, L = Q.attention_int8(qi, qs, ki, ks, vi, vs, False, 1 / 8)
    Oe, Le = A.attention(x, y, z, False, 1 / 8)
    assert np.abs(O - Oe).max() < 0.05 and np.abs(L - Le).max() < 0.02
    cos = (O * Oe).sum() / np.linalg.norm(O) / np.linalg.norm(Oe)
    assert cos > 0.999


def test_int8_single_visible_key_is_exact_value_row():
    x, y, z = (RNG.standard_normal((1, 1, n, 16)) for n in (6, 6, 6))
    qi, qs = Q.quantize_int8_rows(x)
    ki, ks = Q.quantize_int8_rows(y)
    vi, vs = Q.quantize_int8_heads(z)
    O, _ = Q.attention_int8(qi, qs, ki, ks, vi, vs, True, 0.3)
    np.testing.assert_allclose(O[0, 0, 0], vi[0, 0, 0] * float(vs[0, 0]), atol=1e-12)


# ----------------------------------------------------------------- FP4 ------

def test_e2m1_table_matches_spec():
    for code, val in _table("e2m1_values.txt"):
        got = Q.e2m1_decode(code)
        assert got == val and (np.signbit(got) == np.signbit(val) or val == 0)
        assert Q.e2m1_encode(np.array(val)) == (code if code != 8 else 0)


def test_e2m1_encode_nearest_ties_even_and_saturates():
    mids = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for x, c in mids.items():
        assert Q.e2m1_encode(np.array(x)) == c
        assert Q.e2m1_encode(np.array(-x)) == (c + 8 if c else 0)
    assert Q.e2m1_encode(np.array(1e9)) == 7 and Q.e2m1_encode(np.array(-7.0)) == 15
    xs = np.linspace(-7, 7, 20001)
    dec = Q.e2m1_decode(Q.e2m1_encode(xs))
    best = np.abs(np.clip(xs, -6, 6)[:, None] - np.concatenate([Q.E2M1_VALUES, -Q.E2M1_VALUES])).min(1)
    np.testing.assert_allclose(np.abs(dec - np.clip(xs, -6, 6)), best, atol=1e-15)


def test_e4m3_table_matches_spec_and_roundtrips():
    for code, val in _table("e4m3_values.txt"):
        assert Q.ue4m3_decode(code) == val
        assert Q.ue4m3_encode(np.array(val)) == code
    codes = np.arange(127)
    assert np.array_equal(Q.ue4m3_encode(Q.ue4m3_decode(codes)), codes)
    assert (np.diff(Q.UE4M3_VALUES) > 0).all()
    assert Q.ue4m3_encode(np.array(1e6)) == 0x7E


def test_e4m3_ties_to_even():
    v = Q.UE4M3_VALUES
    mid = (v[1:] + v[:-1]) / 2
    got = Q.ue4m3_encode(mid)
    lo = np.arange(126)
    want = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(got, want)


def test_nvfp4_identity_on_grid_with_block_amax_6():
    vals = np.concatenate([Q.E2M1_VALUES, -Q.E2M1_VALUES])
    x = RNG.choice(vals, size=(2, 3, 16, 64))
    x[..., ::16] = 6.0
    codes, sf = Q.quantize_nvfp4(x, axis=-1)
    assert (sf == 0x38).all()
    np.testing.assert_array_equal(Q.nvfp4_dequantize(codes, sf, axis=-1), x)
    codes_t, sf_t = Q.quantize_nvfp4(np.swapaxes(x, -1, -2), axis=-2)
    np.testing.assert_array_equal(Q.nvfp4_dequantize(codes_t, sf_t, axis=-2), np.swapaxes(x, -1, -2))


def test_nvfp4_error_bound_and_zero_block():
    x = RNG.standard_normal((4, 64)) * 5
    x[1, 16:32] = 0.0
    codes, sf = Q.quantize_nvfp4(x)
    assert sf[1, 1] == 0 and (codes[1, 16:32] == 0).all()
    deq = Q.nvfp4_dequantize(codes, sf)
    s = np.repeat(Q.ue4m3_decode(sf), 16, axis=-1)
    # the e2m1 grid has spacing <= 2 below 6: error <= s (half of 2 * s), plus
    # saturation when amax/6 rounds the scale down (<= 1/16 relative)
    assert (np.abs(deq - x) <= s * 1.0 + np.abs(x) / 15 + 1e-12).all()


def test_direct_p_equals_threshold_rule():
    """Direct-P as thresholds on x' (the e2m1 midpoints t mapped back through
    log2(t / 6)) gives the same code as rounding 6 * 2^x' -- away from exact
    ties, which only x' = -3 (t = 0.75) can hit."""
    xp = np.linspace(-8, 0, 400001)
    vals, codes = Q.direct_p_values(xp)
    t = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    thr = np.log2(t / 6.0)
    code_thr = (xp[:, None] > thr).sum(1)
    exact = np.isclose(xp, -3.0, atol=0)
    assert np.array_equal(np.where(exact, codes, code_thr), codes)
    assert Q.direct_p_values(np.array([-3.0]))[1][0] == 2          # tie at 0.75 -> even code 2
    assert Q.direct_p_values(np.array([0.0]))[0][0] == 6.0
    assert Q.direct_p_values(np.array([-np.inf]))[0][0] == 0.0


def test_quant_after_exp_scale_and_codes():
    p = np.exp2(-np.abs(RNG.standard_normal((3, 32))) * 3)
    p[0, :16] = 0.0
    deq, codes, sf = Q.quant_after_exp_values(p)
    assert sf[0, 0] == 0 and (deq[0, :16] == 0).all()
    s = np.repeat(Q.ue4m3_decode(sf), 16, axis=-1)
    assert (np.abs(deq - p) <= s + 1e-12).all()


def _fp4_inputs(Nq, Nkv, d, scale_in=1.0):
    x = RNG.standard_normal((1, 2, Nq, d)) * scale_in
    y = RNG.standard_normal((1, 2, Nkv, d)) * scale_in
    z = RNG.standard_normal((1, 2, Nkv, d))
    qc, qsf = Q.quantize_nvfp4(x, axis=-1)
    kc, ksf = Q.quantize_nvfp4(y, axis=-1)
    vc, vsf = Q.quantize_nvfp4(z, axis=-2)
    return (x, y, z, Q.nvfp4_dequantize(qc, qsf, -1), Q.nvfp4_dequantize(kc, ksf, -1),
            Q.nvfp4_dequantize(vc, vsf, -2))


@pytest.mark.parametrize("mode", [Q.DIRECT_P, Q.QUANT_AFTER_EXP])
def test_fp4_emulation_brute_force(mode):
    *_, qd, kd, vd = _fp4_inputs(3, 32, 16)
    O, L = Q.attention_fp4(qd, kd, vd, mode, False, 0.5, Bc=16)
    for i in range(3):
        m, l, acc = -math.inf, 0.0, np.zeros(16)
        for j0 in range(0, 32, 16):
            x = [float(qd[0, 0, i] @ kd[0, 0, j]) * 0.5 / math.log(2) for j in range(j0, j0 + 16)]
            mb = max(x)
            if mb > m:
                f = 0.0 if m == -math.inf else 2.0 ** (m - mb)
                acc, l, m = acc * f, l * f, mb
            if mode == Q.DIRECT_P:
                pt = [Q.e2m1_decode(Q.e2m1_encode(np.array(6 * 2.0 ** (xx - m)))) / 6 for xx in x]
            else:
                p = np.array([2.0 ** (xx - m) for xx in x], dtype=np.float32)
                sf = Q.ue4m3_decode(Q.ue4m3_encode(np.float32(p.max()) / np.float32(6)))
                pt = [Q.e2m1_decode(Q.e2m1_encode(np.float32(pp) / np.float32(sf))) * sf for pp in p]
            for jj, w in enumerate(pt):
                l += float(w)
                acc = acc + float(w) * vd[0, 0, j0 + jj]
        np.testing.assert_allclose(O[0, 0, i], acc / l, atol=1e-12)
        np.testing.assert_allclose(L[0, 0, i], math.log(2) * (m + math.log2(l)), atol=1e-12)


@pytest.mark.parametrize("mode", [Q.DIRECT_P, Q.QUANT_AFTER_EXP])
def test_fp4_emulation_tracks_exact_attention(mode):
    x, y, z, qd, kd, vd = _fp4_inputs(32, 256, 64)
    O, _ = Q.attention_fp4(qd, kd, vd, mode, False, 1 / 8)
    Oe, _ = A.attention(x, y, z, False, 1 / 8)
    cos = (O * Oe).sum() / np.linalg.norm(O) / np.linalg.norm(Oe)
    assert cos > 0.9
    # with exact (dequantised) operands only P's quantisation remains
    Od, _ = A.attention(qd, kd, vd, False, 1 / 8)
    assert np.abs(O - Od).max() < 0.5


def test_fp4_single_visible_key():
    *_, qd, kd, vd = _fp4_inputs(16, 16, 16)
    for mode in (Q.DIRECT_P, Q.QUANT_AFTER_EXP):
        O, _ = Q.attention_fp4(qd, kd, vd, mode, True, 0.3)
        np.testing.assert_allclose(O[0, :, 0], vd[0, :, 0], atol=1e-12)


# ---------------------------------------------------------------- INT4 Q/K
def test_int4_rows_identity_on_integer_rows_with_amax_7():
    """Rows of integers in [-7, 7] whose amax is 7: s = 7 / 7 = 1 exactly, so
    quantisation is the identity."""
    g = np.random.default_rng(4)
    x = g.integers(-7, 8, size=(3, 5, 16)).astype(np.float32)
    x[..., 0] = 7.0
    q, s = Q.quantize_int4_rows(torch.tensor(x).to(torch.bfloat16))
    assert (s == 1.0).all() and np.array_equal(q.astype(np.float32), x)


def test_int4_rows_zero_row_error_bound_and_range():
    g = torch.Generator().manual_seed(6)
    x = torch.randn(2, 3, 40, 64, generator=g).to(torch.bfloat16)
    x[0, 0, 3] = 0
    q, s = Q.quantize_int4_rows(x)
    assert q[0, 0, 3].tolist() == [0] * 64 and s[0, 0, 3] == 1.0
    assert q.min() >= -7 and q.max() <= 7
    xf = x.double().numpy()
    err = np.abs(xf - q.astype(np.float64) * s[..., None].astype(np.float64))
    assert (err <= 0.5 * s[..., None] * (1 + 1e-6)).all()
    # every row uses the full range: its largest magnitude maps to +-7
    assert (np.abs(q).max(axis=-1)[s != 1.0] == 7).all()


def test_int4_emulation_drifts_more_than_int8_but_stays_close():
    """The same emulated forward with INT4 Q/K: further from the exact
    attention than with INT8 Q/K, still close on N(0,1) inputs."""
    g = torch.Generator().manual_seed(9)
    q, k, v = (torch.randn(1, 2, 96, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    Oe, _ = A.attention(q, k, v, False, 0.125)
    vi, vs = Q.quantize_int8_heads(v)
    errs = []
    for quant in (Q.quantize_int8_rows, Q.quantize_int4_rows):
        qi, qs = quant(q)
        ki, ks = quant(k)
        O, _ = Q.attention_int8(qi, qs, ki, ks, vi, vs, False, 0.125)
        errs.append(np.abs(O - Oe).max())
    assert errs[0] < errs[1] < 0.25
