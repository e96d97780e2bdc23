"""Pins of the FP8 (e4m3) oracle with incoherent processing (oracle/fp8.py)
against what the format definition and the mathematics fix."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import fp8 as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_fwht_equals_sylvester_hadamard_product():
    """On small integers every fp32 sum is exact, so the staged transform must
    equal the explicit H_d x product exactly."""
    g = np.random.default_rng(1)
    for d in (64, 128):
        x = g.integers(-50, 51, size=(7, d)).astype(np.float32)
        assert np.array_equal(F.fwht_f32(x).astype(np.float64), x.astype(np.float64) @ F.hadamard(d).T)


def test_fwht_twice_is_d_times_identity_and_preserves_dot_products():
    g = np.random.default_rng(2)
    d = 128
    x = g.integers(-20, 21, size=(5, d)).astype(np.float32)
    assert np.array_equal(F.fwht_f32(F.fwht_f32(x)), (d * x).astype(np.float32))
    sigma = np.where(g.random(d) < 0.5, -1.0, 1.0).astype(np.float32)
    q, k = x[0:2], x[2:4]
    rq, rk = F.fwht_f32(q * sigma), F.fwht_f32(k * sigma)
    # (H diag(s) q) . (H diag(s) k) = d (q . k): the forward divides by d
    assert np.array_equal(rq.astype(np.float64) @ rk.T.astype(np.float64), d * (q.astype(np.float64) @ k.T))


def test_e4m3_encode_against_the_format_table():
    for line in open(os.path.join(GOLDEN, "e4m3_values.txt")):
        if line.startswith("#") or not line.strip():
            continue
        _, val = line.split()
        v = float(val)
        assert F.e4m3_encode_value(v) == v and F.e4m3_encode_value(-v) == -v
    # every finite value maps to itself; the midpoint between neighbours goes to the even code
    vals = F.UE4M3_VALUES
    assert np.array_equal(F.e4m3_encode_value(vals), vals)
    mids = (vals[:-1] + vals[1:]) / 2
    got = F.e4m3_encode_value(mids)
    even = np.where(np.arange(len(vals) - 1) % 2 == 0, vals[:-1], vals[1:])
    assert np.array_equal(got, even)
    # saturation
    assert F.e4m3_encode_value(1e6) == 448.0 and F.e4m3_encode_value(-500.0) == -448.0


def test_fp8_rows_identity_on_grid_with_amax_448():
    g = np.random.default_rng(3)
    vals = F.UE4M3_VALUES
    x = g.choice(vals, size=(4, 64)) * np.where(g.random((4, 64)) < 0.5, -1, 1)
    x[:, 0] = 448.0
    q, s = F.quantize_fp8_rows(torch.tensor(x, dtype=torch.float32))
    assert (s == 1.0).all() and np.array_equal(q, x)


def test_fp8_channel_scales_and_error_bound():
    g = torch.Generator().manual_seed(4)
    v = torch.randn(1, 2, 300, 64, generator=g).to(torch.bfloat16)
    v[0, 1, :, 5] = 0
    q, s = F.quantize_fp8_channels(v)
    assert s.shape == (1, 2, 64) and s[0, 1, 5] == 1.0 and (q[0, 1, :, 5] == 0).all()
    vf = v.double().numpy()
    rel = np.abs(q * s[:, :, None, :] - vf) / np.maximum(np.abs(vf), 2.0 ** -6 * s[:, :, None, :])
    assert rel.max() <= 2.0 ** -4 * (1 + 1e-6)          # half an e4m3 step (3 mantissa bits)


def test_single_visible_key_gives_the_quantised_value_row():
    """Causal row 0 sees key 0 only: P~ = e4m3(1) = 1 and O = deq(V)[0]."""
    g = torch.Generator().manual_seed(5)
    q, k, v = (torch.randn(1, 1, 16, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    qv, qs = F.quantize_fp8_rows(q)
    kv, ks = F.quantize_fp8_rows(k)
    vv, vs = F.quantize_fp8_channels(v)
    O, L = F.attention_fp8(qv, qs, kv, ks, vv, vs, True, 0.125)
    assert np.array_equal(O[0, 0, 0], vv[0, 0, 0] * vs[0, 0])


def test_rotation_reduces_fp8_error_on_outlier_inputs():
    """The page's point: with a few large channels, rotating Q and K before
    the quantisation lowers the error against the exact attention."""
    from workloads import make_qkv
    q, k, v = make_qkv("lowp", seed=3, B=1, H=2, Nq=256, Nkv=384, d=128)
    Oe, _ = A.attention(q, k, v, False, 128 ** -0.5)
    vv, vs = F.quantize_fp8_channels(v)
    errs = []
    for signs in (None, np.where(np.random.default_rng(7).random(128) < 0.5, -1.0, 1.0)):
        qv, qs = F.quantize_fp8_rows(q, signs)
        kv, ks = F.quantize_fp8_rows(k, signs)
        O, _ = F.attention_fp8(qv, qs, kv, ks, vv, vs, False, 128 ** -0.5, rot_d=128 if signs is not None else 1)
        errs.append(np.abs(O - Oe).max())
    assert errs[1] < errs[0]


def test_fp8_emulation_close_to_exact_attention():
    g = torch.Generator().manual_seed(6)
    q, k, v = (torch.randn(1, 2, 200, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    Oe, Le = A.attention(q, k, v, True, 0.125)
    signs = np.where(np.random.default_rng(8).random(64) < 0.5, -1.0, 1.0)
    qv, qs = F.quantize_fp8_rows(q, signs)
    kv, ks = F.quantize_fp8_rows(k, signs)
    vv, vs = F.quantize_fp8_channels(v)
    O, L = F.attention_fp8(qv, qs, kv, ks, vv, vs, True, 0.125, rot_d=64)
    cos = (O * Oe).sum() / (np.linalg.norm(O) * np.linalg.norm(Oe))
    # P in e4m3 (3 mantissa bits) moves l, hence LSE, by a few per cent at most
    assert cos > 0.995 and np.abs(L - Le).max() < 0.1


@pytest.mark.parametrize("tau", [0.0, 8.0])
def test_integer_scores_are_exact_for_every_tau(tau):
    """Base-2 scores that are integers: every P~ = 2^(x - m) the recurrence
    forms (x - m in [-9, 8]) is an e4m3 value, so the blockwise emulation with
    either threshold must equal the softmax definition 2^S / sum 2^S exactly
    (up to fp64 rounding).  The patterns make the reference move inside later
    blocks, stay stale by up to 7 (tau = 8), and jump past the threshold."""
    pat = np.array([[0, 1, 0, 2, 3, 9, 1, 0, 11, 2, 4, 9, 5, 6, 3, 10],
                    [10, 9, 8, 7, 6, 5, 4, 3, 2, 1, 4, 8, 12, 3, 11, 9]], dtype=np.float64)
    N = pat.shape[1]
    qv = np.eye(2)[None, None]                      # row c picks pattern c
    kv = pat.T[None, None]                          # S[c, j] = pat[c, j]
    g = np.random.default_rng(3)
    vv = F.UE4M3_VALUES[g.integers(0, 100, size=(1, 1, N, 2))] * np.where(g.random((1, 1, N, 2)) < 0.5, -1, 1)
    one = np.ones((1, 1, 2), np.float32)
    O, L = F.attention_fp8(qv, one, kv, np.ones((1, 1, N), np.float32), vv, one, False, math.log(2.0),
                           rot_d=1, Bc=4, tau=tau)
    w = 2.0 ** pat
    Oe = (w @ vv[0, 0]) / w.sum(axis=1)[:, None]
    np.testing.assert_allclose(O[0, 0], Oe, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(L[0, 0], np.log(w.sum(axis=1)), rtol=0, atol=1e-13)


def test_lazy_threshold_changes_only_the_rounding():
    """On random rotated inputs tau = 8 and tau = 0 differ only through where
    P~ is rounded: both stay within the e4m3 error of each other."""
    g = np.random.default_rng(5)
    q = g.standard_normal((1, 2, 64, 128)).astype(np.float32)
    k = g.standard_normal((1, 2, 512, 128)).astype(np.float32)
    v = g.standard_normal((1, 2, 512, 128)).astype(np.float32)
    sg = np.where(g.random(128) < 0.5, -1.0, 1.0)
    a = F.quantize_fp8_rows(q, sg) + F.quantize_fp8_rows(k, sg) + F.quantize_fp8_channels(v)
    O0, L0 = F.attention_fp8(*a, False, 128 ** -0.5, rot_d=128, tau=0.0)
    O8, L8 = F.attention_fp8(*a, False, 128 ** -0.5, rot_d=128, tau=8.0)
    assert np.abs(O0 - O8).max() < 0.02 and np.abs(L0 - L8).max() < 0.01
