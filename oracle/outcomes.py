"""Boundary flips of quantised probabilities, and the range of outputs they allow.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The quantised forwards round a probability-like value y to a grid:

* [INT-FA] INT8:                 y = 127 * 2^(x - m)  to the integers 0..127;
* [FP4-FA4] Direct-P:            y = 6 * 2^(x - m)    to the e2m1 values;
* [FP4-FA4] quantise-after-exp:  a = amax(p) / 6      to the e4m3 values (the
                                 block scale sf), then y = p / sf to e2m1;
* FP8 ([FA-trading] "FA3" item 3): y = 2^(x - m)      to the e4m3 values;
* the FP8-P backward ([FP4-FA4]): y = P               to the e4m3 values.

The oracle evaluates x - m and 2^x in float64.  A device evaluates them in
fp32 with an approximate exp2, so where the exact y lies closer to a rounding
midpoint than that evaluation error, either neighbour of the midpoint is a
correct rounding of what the device computed, and the device may take either.
Everywhere else both sides round alike.  These elements are "flagged"; the
pages fix no evaluation precision, so the error model is a reading:

    |device (x - m) - exact (x - m)| <= EVAL_REL * (|x| + |m| + 1)
    device exp2, and one product or reciprocal after it: relative 2^-20

which is about 16 fp32 ulps of the operands; ``eval_band`` turns it into a
half-width around y.

Both outcomes of every flagged element are then admitted: the output a device
may legitimately produce is the exact result for SOME choice of neighbour at
every flagged element (or, where a block scale is flagged, for some choice of
scale and codes for that block).  For an output element

    O_c = (acc_c + sum_v a_vc) / (l + sum_v b_v),

where each flagged "variable" v contributes nothing (the oracle's own
rounding) or one of its options (a_v, b_v) -- the change of the accumulator
and of the row sum that option causes -- the extremes over all choices are
computed exactly by ``ratio_range`` (Dinkelbach's parametric method for a
ratio of linear functions over a finite product set).  A device value is
checked against the interval [min, max] it spans, with the tolerance the
method states and nothing added.  Rows without a flagged element get an
interval of width zero, i.e. the plain check.
"""
from __future__ import annotations

from dataclasses import dataclass
from itertools import combinations

import numpy as np

LN2 = float(np.log(2.0))
EVAL_REL = 2e-6
EXP2_REL = 2.0 ** -20


def eval_band(y, x, m, abs_eps):
    """Half-width of the interval around the exact y = c * 2^(x - m) inside
    which a device's fp32 evaluation may fall (the error model of the module
    docstring), plus ``abs_eps`` for values near zero."""
    dx = EVAL_REL * (np.abs(x) + np.abs(m) + 1.0)
    return np.abs(y) * (LN2 * dx + EXP2_REL) + abs_eps


def near_midpoint(y, grid, base, band):
    """Flag the values y that lie within ``band`` of a rounding midpoint of
    ``grid`` (sorted, non-negative values), and give the other neighbour.

    ``base`` is the grid value the oracle rounded y to.  For a flagged y the
    midpoint between grid[k] and grid[k + 1] is the nearest one, and ``alt``
    is whichever of the two is not ``base``.  Returns (flag bool, alt float64;
    alt = base where not flagged)."""
    y = np.asarray(y, dtype=np.float64)
    g = np.asarray(grid, dtype=np.float64)
    mids = (g[1:] + g[:-1]) / 2.0
    i = np.clip(np.searchsorted(mids, y), 0, mids.size - 1)
    lo = np.clip(i - 1, 0, mids.size - 1)
    pick = np.where(np.abs(y - mids[lo]) < np.abs(y - mids[i]), lo, i)
    dist = np.abs(y - mids[pick])
    flag = dist <= band
    below, above = g[pick], g[pick + 1]
    alt = np.where(base == below, above, below)
    return flag, np.where(flag, alt, base)


def ratio_range(num, den, opt_a, opt_b, max_iter=200):
    """Exact minimum and maximum of

        (num_c + sum_v a_vc) / (den + sum_v b_v)

    over every choice in which each variable v contributes either nothing or
    one of its options k: (a_v, b_v) = (opt_a[v, k], opt_b[v, k]).  ``num`` is
    [d] (independent columns c sharing the denominator; each column gets its
    own extremes), ``den`` a scalar, ``opt_a`` [V, K, d], ``opt_b`` [V, K]
    (pad missing options with zeros: an all-zero option is the same as
    contributing nothing).  Needs den + sum_v min(0, min_k b_vk) > 0.

    Method (Dinkelbach): for the current value lam, the choice minimising
    N - lam * D takes, per variable, the option with the smallest
    a - lam * b if that is negative, else nothing; the new lam = N / D of that
    choice.  lam decreases strictly until the choice repeats, at which point
    min (N - lam D) = 0, i.e. lam = min N / D.  The maximum is the same with
    the signs reversed.  Returns (lo [d], hi [d])."""
    num = np.asarray(num, dtype=np.float64)
    opt_a = np.asarray(opt_a, dtype=np.float64)
    opt_b = np.asarray(opt_b, dtype=np.float64)
    base = num / den
    V = opt_b.shape[0]
    if V == 0:
        return base.copy(), base.copy()
    dmin = den + np.minimum(opt_b.min(axis=1), 0.0).sum()
    if not dmin > 0:
        raise ValueError("a choice of outcomes makes the row sum non-positive")
    vi = np.arange(V)[:, None]
    out = []
    for sgn in (1.0, -1.0):
        lam = base.copy()
        prev = None
        for _ in range(max_iter):
            val = sgn * (opt_a - lam[None, None, :] * opt_b[:, :, None])        # [V, K, d]
            k = val.argmin(axis=1)                                            # [V, d]
            best = np.take_along_axis(val, k[:, None, :], axis=1)[:, 0, :]
            take = best < 0
            a = np.where(take, np.take_along_axis(opt_a, k[:, None, :], axis=1)[:, 0, :], 0.0).sum(axis=0)
            b = np.where(take, opt_b[vi, k], 0.0).sum(axis=0)
            sel = np.where(take, k, -1)
            if prev is not None and np.array_equal(sel, prev):
                break
            prev = sel
            lam = (num + a) / (den + b)
        out.append(lam)
    return out[0], out[1]


@dataclass
class OutcomeRange:
    """Interval of the outputs that every admissible rounding of the flagged
    elements gives: O_lo <= O <= O_hi and LSE_lo <= LSE <= LSE_hi elementwise
    (float64, the shapes of O and LSE).  ``flips`` counts flagged variables
    (elements, or blocks whose scale is flagged), ``flagged_rows`` the query
    rows holding at least one, ``rows`` all query rows."""
    O_lo: np.ndarray
    O_hi: np.ndarray
    LSE_lo: np.ndarray
    LSE_hi: np.ndarray
    flips: int
    flagged_rows: int
    rows: int
    ambiguous_rescales: int = 0

    def distance(self, O, LSE):
        """How far device outputs lie outside the interval (0 inside):
        (max over O elements, max over finite-LSE rows)."""
        O = np.asarray(O, dtype=np.float64)
        dO = np.maximum(np.maximum(self.O_lo - O, O - self.O_hi), 0.0)
        fin = np.isfinite(self.LSE_lo)
        L = np.asarray(LSE, dtype=np.float64)
        dL = np.maximum(np.maximum(self.LSE_lo[fin] - L[fin], L[fin] - self.LSE_hi[fin]), 0.0)
        return float(dO.max(initial=0.0)), float(dL.max(initial=0.0))

    def width(self):
        """Largest O interval width (0 when nothing is flagged)."""
        return float((self.O_hi - self.O_lo).max(initial=0.0))


class FlipRecorder:
    """The flagged variables of one (batch, head) slice of a blockwise
    quantised forward.  A variable is one element with one alternative value,
    or a group of keys (a block) with several alternative value vectors.
    Deltas are in the units of the quantised P (before any later rescale);
    ``m_blk`` is the reference max the block was quantised against."""

    def __init__(self):
        self.vars = {}            # row -> list of (keys int[n], options [K, n], m_blk)

    def add_elements(self, rows, keys, delta, m_blk):
        for r, j, dl, mb in zip(np.asarray(rows).ravel(), np.asarray(keys).ravel(),
                                np.asarray(delta, dtype=np.float64).ravel(), np.asarray(m_blk).ravel()):
            self.vars.setdefault(int(r), []).append((np.array([int(j)]), np.array([[dl]]), float(mb)))

    def add_group(self, row, keys, options, m_blk):
        opts = np.asarray(options, dtype=np.float64)
        if opts.size and np.any(opts != 0):
            self.vars.setdefault(int(row), []).append((np.asarray(keys, dtype=np.int64), opts, float(m_blk)))

    def count(self):
        return sum(len(v) for v in self.vars.values())

    def intervals(self, num, l, m_final, U, w):
        """Per row r: O = num[r] / l[r] with num = sum_j P~_j f_j U_j and
        l = sum_j P~_j f_j w, f_j = 2^(m_blk(j) - m_final[r]) the rescale of
        key j's block to the final reference.  Returns (O_lo, O_hi, l_lo,
        l_hi) for every row (width zero where nothing is flagged)."""
        R, d = num.shape
        ok = l > 0
        ls = np.where(ok, l, 1.0)
        O = np.where(ok[:, None], num / ls[:, None], 0.0)
        O_lo, O_hi = O.copy(), O.copy()
        l_lo, l_hi = l.copy(), l.copy()
        for r, vs in self.vars.items():
            K = max(o.shape[0] for _, o, _ in vs)
            A = np.zeros((len(vs), K, d))
            Bv = np.zeros((len(vs), K))
            for v, (keys, opts, mb) in enumerate(vs):
                f = 2.0 ** (mb - m_final[r])
                A[v, :opts.shape[0]] = f * (opts @ U[keys])
                Bv[v, :opts.shape[0]] = f * w * opts.sum(axis=1)
            O_lo[r], O_hi[r] = ratio_range(num[r], l[r], A, Bv)
            l_lo[r] = l[r] + np.minimum(Bv.min(axis=1), 0.0).sum()
            l_hi[r] = l[r] + np.maximum(Bv.max(axis=1), 0.0).sum()
        return O_lo, O_hi, l_lo, l_hi


def subset_options(base_vals, alt_vals, flagged):
    """All non-empty subsets of the flagged positions switched from their base
    value to their alternative: an array [2^f - 1, n] of deltas (n = len(base))."""
    idx = np.flatnonzero(flagged)
    n = len(base_vals)
    out = []
    for size in range(1, idx.size + 1):
        for sub in combinations(idx.tolist(), size):
            d = np.zeros(n)
            d[list(sub)] = alt_vals[list(sub)] - base_vals[list(sub)]
            out.append(d)
    return np.array(out).reshape(-1, n)
