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
from .lowp import UE4M3_VALUES, _near_half  # noqa: F401  (value table of the format)

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


def attention_fp8(qv, qs, kv, ks, vv, vs, causal=False, scale=None, rot_d=1, Bc=128,
                  with_flip_bound=False, rows=None, tau=0.0):
    """Emulated FP8 forward (steps 3-5 of the module docstring) from code values
    and scales; ``rot_d`` = d when Q and K were rotated (the product is then d
    times Q K^T), 1 otherwise.  Returns (O, LSE) float64 and, with
    ``with_flip_bound``, (flip_bound, lse_flip_bound, flips): how far O and
    LSE can move if a P element within fp32 evaluation error of an e4m3
    rounding midpoint rounds the other way on the device."""
    qv, kv, vv = _f64(qv), _f64(kv), _f64(vv)
    B, H, Nq_all, d = qv.shape
    Nkv = kv.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ridx = np.arange(Nq_all) if rows is None else np.asarray(rows)
    Nq = ridx.size
    O = np.zeros((B, H, Nq, d))
    LSE = np.full((B, H, Nq), -np.inf)
    FB = np.zeros((B, H, Nq, d))
    LB = np.zeros((B, H, Nq))
    flips = 0
    vis = visible_mask(Nq_all, Nkv, causal, ridx)
    # e4m3 rounding midpoints up to the largest P~ (2^tau): the value between two neighbours
    mids = (UE4M3_VALUES[:-1] + UE4M3_VALUES[1:]) / 2.0
    mids = mids[mids <= 2.0 ** tau * 1.07]
    for b in range(B):
        for h in range(H):
            S = (qv[b, h, ridx] @ kv[b, h].T).astype(F32).astype(np.float64)
            x = S * (_f64(qs)[b, h, ridx][:, None] * _f64(ks)[b, h][None, :]) * (scale * LOG2E / rot_d)
            x = np.where(vis, x, -np.inf)
            acc = np.zeros((Nq, d))
            l = np.zeros(Nq)
            m = np.full(Nq, -np.inf)
            wflip = np.zeros((Nq, Nkv))
            for j0 in range(0, Nkv, Bc):
                cols = slice(j0, min(Nkv, j0 + Bc))
                xb = x[:, cols]
                m_new = np.maximum(m, xb.max(axis=1))
                move = np.isfinite(m_new) & (~np.isfinite(m) | (m_new > m + tau))
                grow = move & np.isfinite(m)
                f = np.ones_like(m)
                with np.errstate(invalid="ignore"):  # -inf - -inf where not grow (not used)
                    np.exp2(m - m_new, out=f, where=grow)
                acc *= f[:, None]
                l *= f
                m = np.where(move, m_new, m)
                ms = np.where(np.isfinite(m), m, 0.0)
                fin = np.isfinite(xb) & np.isfinite(m)[:, None]
                p = np.zeros_like(xb)
                np.exp2(np.where(fin, xb - ms[:, None], 0.0), out=p, where=fin)
                P = e4m3_encode_value(p)
                if with_flip_bound:
                    # fp32 evaluation of x and of exp2: a few ulps of |x|, |m|
                    dx = 2e-6 * (np.abs(np.where(fin, xb, 0.0)) + np.abs(ms)[:, None] + 1.0)
                    band = p * LN2 * dx + 1e-7
                    near = np.zeros_like(p, dtype=bool)
                    for t in mids:
                        near |= np.abs(p - t) < band
                    near &= fin
                    # a flip moves P by one e4m3 step: at most 2^-3 * P (normal) or 2^-9
                    step = np.maximum(p * 0.125, 2.0 ** -9)
                    wflip[:, cols] = np.where(near, step, 0.0)
                l += P.sum(axis=1)
                acc += P @ vv[b, h, cols]
            ok = l > 0
            ls = np.where(ok, l, 1.0)
            sv = _f64(vs)[b, h]
            O[b, h] = np.where(ok[:, None], acc * sv[None, :] / ls[:, None], 0.0)
            LSE[b, h] = np.where(ok, LN2 * (np.where(ok, m, 0.0) + np.log2(ls)), -np.inf)
            if with_flip_bound:
                flips += int(np.count_nonzero(wflip))
                vdeq = vv[b, h] * sv[None, :]
                FB[b, h] = (wflip @ np.abs(vdeq) + wflip.sum(axis=1)[:, None] * np.abs(O[b, h])) / ls[:, None]
                LB[b, h] = wflip.sum(axis=1) / ls * 1.01
    if with_flip_bound:
        return O, LSE, FB, LB, flips
    return O, LSE
