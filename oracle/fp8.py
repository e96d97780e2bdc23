"""Quantisers and step-by-step emulation of the FP8 (e4m3) attention forward
with incoherent processing.

TEST INFRASTRUCTURE ONLY (see the package docstring).

[FA-trading] "FA2"/"FA3" list, item 3 (FP8 with incoherent processing): FP8
runs at twice the FP16 rate, naive FP8 attention is broken by outliers, and
FA3 randomly rotates the vectors before block quantisation so that an
outlier's magnitude is spread over the coordinates.  The page names the idea,
not the formulas; the readings taken here:

  1. Rotation of Q and K rows (along d): y = H_d (sigma o x), sigma in
     {+1, -1}^d a seeded sign vector passed in as an input, H_d the Sylvester
     Hadamard matrix (entries +-1, unnormalised), evaluated as the fast
     Walsh-Hadamard transform in fp32: stages h = 1, 2, 4, ..., d/2, each
     replacing the pair (a, b) = (y[e], y[e + h]) (bit h of e clear) by
     (a + b, a - b).  H_d H_d^T = d I, so (Q R)(K R)^T = d Q K^T and the
     forward divides the softmax scale by d (exact: d is a power of two).  V
     is not rotated.
  2. e4m3 (OCP 8-bit floating point E4M3: bias 7, three mantissa bits,
     subnormals, largest finite 448), round to nearest even, saturating.
     Q, K: one fp32 scale per token row, s = amax / 448 (IEEE fp32 divide),
     code = e4m3(y / s) (IEEE fp32 divide); V: one scale per channel over a
     head's tokens (P V contracts over tokens; a channel scale factors out of
     the product), s_c = amax_j |v_jc| / 448.  A zero amax gives s = 1.
  3. S = sum_c deq(Q)_ic deq(K)_jc without the scales (exact e4m3 products,
     fp64 sum), rounded once to fp32; x = S * s_Q[i] * s_K[j] * scale *
     log2(e) / d, masked.
  4. blockwise over B_c = 128 keys with a reference max m that moves to the
     block max only when that exceeds it by more than tau ([FA4-overview]
     "Smarter online softmax rescaling"; tau = 0 moves it on every increase):
     P~ = e4m3(2^(x - m)) with unit scale, l = l * 2^(m_old - m) + sum P~,
     acc = acc * 2^(m_old - m) + P~ . codes(V).  The FP8 kernel takes tau = 8:
     P~ <= 2^8 = 256 stays inside e4m3's finite range (448), and the precision
     of e4m3 is the same in every binade of its normal range.
  5. O_c = acc_c * s_V[c] / l, LSE = ln2 (m + log2 l).
"""
from __future__ import annotations

import math

import numpy as np

from .attention import LN2, LOG2E, _f64, visible_mask
from .lowp import UE4M3_VALUES, _RangeCollector  # value table of the format; interval collector
from .outcomes import EVAL_REL, FlipRecorder, eval_band, near_midpoint

F32 = np.float32
E4M3_MAX = 448.0


def fwht_f32(x):
    """Unnormalised fast Walsh-Hadamard transform along the last axis, in fp32,
    stage by stage (h = 1, 2, 4, ...; (a, b) -> (a + b, a - b))."""
    y = np.array(x, dtype=F32, copy=True)
    d = y.shape[-1]
    assert d & (d - 1) == 0, "d must be a power of two"
    h = 1
    while h < d:
        z = y.reshape(y.shape[:-1] + (d // (2 * h), 2, h))
        a = z[..., 0, :].copy()
        b = z[..., 1, :].copy()
        z[..., 0, :] = a + b
        z[..., 1, :] = a - b
        y = z.reshape(y.shape)
        h *= 2
    return y


def hadamard(d: int) -> np.ndarray:
    """Sylvester Hadamard matrix H_d (entries +-1), H[i][j] = (-1)^popcount(i & j)."""
    i = np.arange(d)
    return np.where((np.bitwise_count(i[:, None] & i[None, :]) % 2) == 0, 1.0, -1.0)


def e4m3_encode_value(x):
    """Round to the nearest signed e4m3 value (ties to even code), saturating
    at +-448; returns the value (float64).  The sign of a zero is dropped."""
    x = _f64(x)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(UE4M3_VALUES, a, side="left"), 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    dl = np.abs(a - UE4M3_VALUES[lo])
    dh = np.abs(UE4M3_VALUES[hi] - a)
    code = np.where((dh < dl) | ((dh == dl) & (hi % 2 == 0)), hi, lo)
    return np.sign(x) * UE4M3_VALUES[code]


def quantize_fp8_rows(x, signs=None):
    """Q or K: optional rotation by H_d diag(signs) (fp32 FWHT), then e4m3 per
    token row.  Returns (values of the codes [..., d] float64, scales float32)."""
    y = _f64(x).astype(F32)
    if signs is not None:
        y = fwht_f32(y * np.asarray(signs, dtype=F32))
    amax = np.abs(y).max(axis=-1)
    s = (amax / F32(E4M3_MAX)).astype(F32)
    s = np.where(amax == 0, F32(1.0), s).astype(F32)
    q = e4m3_encode_value((y / s[..., None]).astype(F32))
    return q, s


def quantize_fp8_channels(v):
    """V [B,H,N,d]: e4m3 with one scale per (batch, head, channel) over tokens.
    Returns (values of the codes float64, scales float32 [B,H,d])."""
    y = _f64(v).astype(F32)
    amax = np.abs(y).max(axis=-2)
    s = (amax / F32(E4M3_MAX)).astype(F32)
    s = np.where(amax == 0, F32(1.0), s).astype(F32)
    q = e4m3_encode_value((y / s[..., None, :]).astype(F32))
    return q, s


def _fp8_rows(x, vvs, tau, Bc, outcomes, invert=None):
    """Steps 4-5 for the rows of one (batch, head): x [R, Nkv] base-2 scores
    (masked = -inf), vvs [Nkv, d] = codes(V) * s_V (the channel scales folded
    in, which is exact in exact arithmetic).  ``invert`` [R, n_blocks] bool
    reverses the lazy-rescale decision of those (row, block) pairs.  Returns
    (num [R, d], l, m, FlipRecorder or None, ambiguous [R, n_blocks])."""
    R, Nkv = x.shape
    nblk = -(-Nkv // Bc)
    num = np.zeros((R, vvs.shape[1]))
    l = np.zeros(R)
    m = np.full(R, -np.inf)
    rec = FlipRecorder() if outcomes else None
    amb = np.zeros((R, nblk), dtype=bool)
    for jb, j0 in enumerate(range(0, Nkv, Bc)):
        cols = slice(j0, min(Nkv, j0 + Bc))
        xb = x[:, cols]
        m_blk = xb.max(axis=1)
        m_new = np.maximum(m, m_blk)
        move = np.isfinite(m_new) & (~np.isfinite(m) | (m_new > m + tau))
        if tau > 0:
            both = np.isfinite(m) & np.isfinite(m_blk)
            mb0, m0 = np.where(both, m_blk, 0.0), np.where(both, m, 0.0)
            amb[:, jb] = both & (np.abs(mb0 - (m0 + tau)) <= EVAL_REL * (np.abs(mb0) + np.abs(m0) + 1.0))
            if invert is not None:
                # the other decision: move to the block max (if the block raises it at all)
                flip = invert[:, jb] & both
                move = np.where(flip, ~move & (m_new > m), move)
        grow = move & np.isfinite(m)
        f = np.ones_like(m)
        with np.errstate(invalid="ignore"):  # -inf - -inf where not grow (not used)
            np.exp2(m - m_new, out=f, where=grow)
        num *= f[:, None]
        l *= f
        m = np.where(move, m_new, m)
        ms = np.where(np.isfinite(m), m, 0.0)
        fin = np.isfinite(xb) & np.isfinite(m)[:, None]
        p = np.zeros_like(xb)
        np.exp2(np.where(fin, xb - ms[:, None], 0.0), out=p, where=fin)
        P = e4m3_encode_value(p)
        if outcomes:
            band = eval_band(p, np.where(fin, xb, 0.0), ms[:, None], 1e-12)
            flag, alt = near_midpoint(p, UE4M3_VALUES, P, band)
            r_, c_ = np.nonzero(flag & fin)
            rec.add_elements(r_, c_ + j0, (alt - P)[r_, c_], ms[r_])
        l += P.sum(axis=1)
        num += P @ vvs[cols]
    return num, l, m, rec, amb


def attention_fp8(qv, qs, kv, ks, vv, vs, causal=False, scale=None, rot_d=1, Bc=128,
                  outcomes=False, rows=None, tau=0.0, max_branches=64):
    """Emulated FP8 forward (steps 3-5 of the module docstring) from code values
    and scales; ``rot_d`` = d when Q and K were rotated (the product is then d
    times Q K^T), 1 otherwise.  Returns (O, LSE) float64 and, with
    ``outcomes``, also an ``OutcomeRange`` over both roundings of every P
    element within fp32 evaluation error of an e4m3 rounding midpoint
    (``oracle.outcomes``).  Where a lazy-rescale decision (block max above
    the reference by more than tau) lies within that error of the threshold,
    a device may decide either way: the row is then followed down both
    decisions (up to ``max_branches`` paths per row) and its interval is the
    hull of theirs; ``ambiguous_rescales`` counts such decisions."""
    qv, kv, vv = _f64(qv), _f64(kv), _f64(vv)
    B, H, Nq_all, d = qv.shape
    Nkv = kv.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ridx = np.arange(Nq_all) if rows is None else np.asarray(rows)
    Nq = ridx.size
    O = np.zeros((B, H, Nq, d))
    LSE = np.full((B, H, Nq), -np.inf)
    rng = _RangeCollector(O.shape) if outcomes else None
    vis = visible_mask(Nq_all, Nkv, causal, ridx)
    for b in range(B):
        for h in range(H):
            S = (qv[b, h, ridx] @ kv[b, h].T).astype(F32).astype(np.float64)
            x = S * (_f64(qs)[b, h, ridx][:, None] * _f64(ks)[b, h][None, :]) * (scale * LOG2E / rot_d)
            x = np.where(vis, x, -np.inf)
            vvs = vv[b, h] * _f64(vs)[b, h][None, :]
            num, l, m, rec, amb = _fp8_rows(x, vvs, tau, Bc, outcomes)
            ok = l > 0
            ls = np.where(ok, l, 1.0)
            O[b, h] = np.where(ok[:, None], num / ls[:, None], 0.0)
            LSE[b, h] = np.where(ok, LN2 * (np.where(ok, m, 0.0) + np.log2(ls)), -np.inf)
            if outcomes:
                rng.add(b, h, rec, num, l, m, vvs, 1.0)
                for r in np.flatnonzero(amb.any(axis=1)):
                    _fp8_branch_hull(rng, b, h, r, x[r:r + 1], vvs, tau, Bc, amb[r], max_branches)
    if outcomes:
        return O, LSE, rng.result(O, LSE)
    return O, LSE


def _fp8_branch_hull(rng, b, h, r, xr, vvs, tau, Bc, amb_r, max_branches):
    """Follow every combination of decisions at the ambiguous blocks of row r
    (new ambiguities found on a branch are followed too) and widen the row's
    interval in ``rng`` to the hull of all branches."""
    nblk = amb_r.size
    seen = set()
    todo = [np.zeros(nblk, dtype=bool)]
    pending = [np.flatnonzero(amb_r)]
    branches = 0
    while todo:
        inv = todo.pop()
        cand = pending.pop()
        for jb in cand:
            nxt = inv.copy()
            nxt[jb] = ~nxt[jb]
            key = nxt.tobytes()
            if key in seen:
                continue
            seen.add(key)
            branches += 1
            if branches > max_branches:
                raise ValueError(f"row {r}: more than {max_branches} lazy-rescale decision paths")
            num, l, m, rec, amb = _fp8_rows(xr, vvs, tau, Bc, True, invert=nxt[None, :])
            lo, hi, llo, lhi = rec.intervals(num, l, m, vvs, 1.0)
            rng.widen(b, h, r, lo[0], hi[0], llo[0], lhi[0], m[0])
            rng.flips += rec.count()
            todo.append(nxt)
            pending.append(np.flatnonzero(amb[0] & ~nxt))
    rng.ambiguous += int(amb_r.sum())
