"""Comparison helpers shared by the GPU parity tests (tolerances in one place).

bf16 path (outputs bf16 O, fp32 LSE): max-abs 2e-2 and mean-abs 2e-3 on O,
1e-3 on LSE, all against the fp64 oracle.  Where |O| is large (inputs with
outlier channels) half an ulp of the bf16 output alone exceeds 2e-2, so the
max-abs bound grows by that half ulp.
"""
import numpy as np
import torch

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def half_ulp_bf16(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)          # bf16: 8 significant bits


def to64(t):
    return t.detach().to("cpu").double().numpy()


def assert_bf16_close(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    o = to64(o_gpu)
    lse = to64(lse_gpu)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.isfinite(o).all(), f"{what}: non-finite O"
    err = np.abs(o - o_ref)
    tol = O_MAX_ABS + half_ulp_bf16(o_ref)
    bad = err > tol
    assert not bad.any(), f"{what}: O max-abs {err.max():.3e} (worst tol {tol[bad].min():.3e}, {bad.sum()} bad)"
    assert err.mean() <= O_MEAN_ABS, f"{what}: O mean-abs {err.mean():.3e}"
    fin = np.isfinite(lse_ref)
    assert (np.isneginf(lse[~fin])).all(), f"{what}: LSE should be -inf for rows that see no key"
    if fin.any():
        le = np.abs(lse[fin] - lse_ref[fin]).max()
        assert le <= LSE_ABS, f"{what}: LSE max-abs {le:.3e}"
    return float(err.max()), float(err.mean())
