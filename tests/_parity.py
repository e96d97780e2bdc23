"""Comparison helpers shared by the GPU parity tests (tolerances in one place).

bf16 path (outputs bf16 O, fp32 LSE): max-abs 2e-2 and mean-abs 2e-3 on O,
1e-3 on LSE, all against the fp64 oracle.

Inputs with outlier channels (|V| up to ~80) need a bound derived from the
arithmetic instead: the kernel rounds every probability to bf16 before P V
(relative error <= 2^-8 per weight, the unit roundoff of an 8-bit significand) and its output to bf16, so

    |O_dev - O|_c <= 2^-8 * sum_j P_j |V_jc| + half a bf16 ulp of |O_c|
                     (+ fp32 accumulation, far smaller),

where sum_j P_j |V_jc| is attention applied to |V| (the oracle computes it).
With ``p_abs_v`` given, max-abs allows 2e-2 plus that bound and mean-abs 2e-3
plus its mean; the error relative to the bound is reported.  For N(0,1)
inputs the bound is below 1e-2 and the plain 2e-2 applies.
"""
import numpy as np

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def half_ulp_bf16(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)          # bf16: 8 significant bits


def to64(t):
    return t.detach().to("cpu").double().numpy()


def bf16_p_bound(o_ref, o_dev, p_abs_v):
    """The arithmetic bound of the module docstring, per element."""
    return 2.0 ** -8 * p_abs_v + half_ulp_bf16(np.maximum(np.abs(o_ref), np.abs(o_dev)))


def assert_bf16_close(o_gpu, lse_gpu, o_ref, lse_ref, what="", p_abs_v=None):
    o = to64(o_gpu)
    lse = to64(lse_gpu)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.isfinite(o).all(), f"{what}: non-finite O"
    err = np.abs(o - o_ref)
    extra = 0.0 if p_abs_v is None else bf16_p_bound(o_ref, o, p_abs_v)
    tol = O_MAX_ABS + extra
    if p_abs_v is not None:
        print(f"{what}: O max-abs {err.max(initial=0):.3e}, mean-abs {err.mean():.3e}; largest error / "
              f"(2^-8 sum P|V| + half ulp) {(err / np.maximum(extra, 1e-30)).max(initial=0):.3f}; "
              f"elements beyond 2e-2 {(err > O_MAX_ABS).sum()}")
    bad = err > tol
    assert not bad.any(), f"{what}: O max-abs {err.max():.3e} (worst tol {np.min(tol[bad]):.3e}, {bad.sum()} bad)"
    mean_tol = O_MEAN_ABS + (0.0 if p_abs_v is None else float(np.mean(extra)))
    assert err.mean() <= mean_tol, f"{what}: O mean-abs {err.mean():.3e} (tol {mean_tol:.3e})"
    fin = np.isfinite(lse_ref)
    assert (np.isneginf(lse[~fin])).all(), f"{what}: LSE should be -inf for rows that see no key"
    if fin.any():
        le = np.abs(lse[fin] - lse_ref[fin]).max()
        assert le <= LSE_ABS, f"{what}: LSE max-abs {le:.3e}"
    return float(err.max()), float(err.mean())


# ------------------------------------------------------------------ quantised paths
Q_O_ABS = 5e-3       # INT8 / FP4 / FP8: max-abs against the emulating oracle
Q_LSE_ABS = 1e-3
MAX_FLIP_RATE = 1e-3  # flagged elements per visible score, asserted per check


def visible_scores(Nq, Nkv, causal, rows=None):
    """Number of (query row, key) pairs that are not masked, per (b, h)."""
    i = np.arange(Nq) if rows is None else np.asarray(rows)
    if not causal:
        return int(i.size) * Nkv
    return int(np.clip(i + (Nkv - Nq) + 1, 0, Nkv).sum())


def assert_within_outcomes(og, lg, O, L, R, what, n_scores, o_abs=Q_O_ABS, lse_abs=Q_LSE_ABS):
    """A quantised forward's device outputs against the emulating oracle.

    ``R`` (oracle.outcomes.OutcomeRange) spans every output the emulation
    gives when each flagged P element (one that lies within fp32 evaluation
    error of a rounding midpoint) takes either neighbour; the device must lie
    within ``o_abs`` of that interval (``lse_abs`` for LSE), nothing added.
    Unflagged rows have an interval of width zero.  The flagged count is
    reported and must stay below MAX_FLIP_RATE of the visible scores
    (``n_scores``, all (b, h) together)."""
    og = np.asarray(og, dtype=np.float64)
    lg = np.asarray(lg, dtype=np.float64)
    assert og.shape == O.shape, (og.shape, O.shape)
    assert np.isfinite(og).all(), f"{what}: non-finite O"
    fin = np.isfinite(L)
    assert np.isneginf(lg[~fin]).all(), f"{what}: LSE should be -inf for rows that see no key"
    dO, dL = R.distance(og, lg)
    plain = float(np.abs(og - O).max(initial=0.0))
    print(f"{what}: flagged rows {R.flagged_rows}/{R.rows}, flagged elements {R.flips} "
          f"({R.flips / max(n_scores, 1):.1e} of {n_scores} scores), widest interval {R.width():.3e}, "
          f"ambiguous rescales {R.ambiguous_rescales}; O outside interval {dO:.3e} "
          f"(vs oracle rounding {plain:.3e}), LSE outside {dL:.3e}")
    assert dO <= o_abs, f"{what}: O {dO:.3e} outside the interval of admissible roundings"
    assert dL <= lse_abs, f"{what}: LSE {dL:.3e} outside the interval of admissible roundings"
    assert R.flips <= MAX_FLIP_RATE * n_scores, f"{what}: {R.flips} flagged elements"
    return dO, plain
