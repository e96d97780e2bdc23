"""Error bound of the FMA-pipe exp2 used for a share of the softmax
exponentials: the kernel's op sequence (magic-add rounding, Horner cubic with
fused multiply-adds, exponent-field add) replayed in fp32 on the CPU against
numpy's exp2.  bf16 P needs a relative error well below 2^-9."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "tiled_attention_24_b200", "csrc", "exp2_poly.cuh")


def coeffs():
    src = open(HDR).read()
    return [np.float32(float.fromhex(re.search(rf"kExp2C{k} = (\S+)f;", src).group(1))) for k in range(4)]


def exp2_poly_fp32(x):
    c0, c1, c2, c3 = coeffs()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    M = np.float32(12582912.0)
    t = (x + M).astype(np.float32)
    f = (x - (t - M).astype(np.float32)).astype(np.float32)

    def fma(a, b, c):
        return (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)
    p = fma(fma(fma(np.full_like(f, c3), f, c2), f, c1), f, c0)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_relative_error_bound_over_softmax_range():
    x = np.linspace(-30.0, 8.0, 2_000_001).astype(np.float32)
    y = exp2_poly_fp32(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.0e-4            # 2^-13.3
    assert rel.max() < 2.0 ** -9 / 8     # far below a bf16 half-ulp


def test_tiny_and_clamped_arguments_stay_positive_and_small():
    x = np.array([-125.0, -200.0, -1e30, -124.5], dtype=np.float32)
    y = exp2_poly_fp32(x)
    assert (y > 0).all() and (y < 1e-37).all()


def test_integers_are_nearly_exact():
    n = np.arange(-100, 9, dtype=np.float32)
    y = exp2_poly_fp32(n).astype(np.float64)
    assert np.abs(y / np.exp2(n.astype(np.float64)) - 1).max() < 1e-4
