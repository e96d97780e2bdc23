"""Quantisers and step-by-step emulations of the INT8 and FP4 attention forwards.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The quantised forwards are not exact methods, so this module follows their
steps in order, in float64 except where a step is defined in fp32 (the
quantisers' divide and round, which the CUDA side must match bit for bit):

INT8 ([INT-FA], token-level post-training quantisation; INT8 GEMMs replace the
floating-point matmuls of the FlashAttention forward):
  1. per-token symmetric scale s = amax(row) / 127 (fp32 divide), q =
     clamp(rne(x / s), -127, 127); an all-zero row gets s = 1, q = 0.
     V uses one scale per (batch, head) (amax over the whole head / 127): P V
     contracts over tokens, so a per-token V scale cannot be taken out of an
     int32 P V product.  This is a reading; the page only says "token-level".
  2. S = q_Q . q_K exactly in integers (int32 range checked).
  3. x = S * s_Q[i] * s_K[j] * scale * log2(e), masked.
  4. blockwise over B_c = 128 keys with the running max moved on every
     increase (tau = 0, so that P never exceeds 1):
       P8 = rne(127 * 2^(x - m)) in [0, 127],
       l  = l * 2^(m_old - m) + sum(P8) / 127,
       acc = acc * 2^(m_old - m) + (P8 . q_V) * s_V / 127.
  5. O = acc / l, LSE = ln2 * (m + log2 l).

FP4 ([FP4-FA4]: FP4 operands; the probabilities either quantised after the
exponential with a scale and rounding, or mapped "directly" to the FP4 codes):
  1. NVFP4: blocks of 16 elements, e2m1 codes with an unsigned e4m3 block
     scale sf = ue4m3_rne(amax / 6), code = e2m1_rne_satfinite(x / sf).  Q and K
     blocks run along d; V blocks run along tokens (P V contracts over tokens).
  2. S = deq(Q) . deq(K) (exact products, fp64 sum), x as above.
  3. blockwise (B_c = 128, tau = 0); per block, x' = x - m <= 0 and
       Direct-P:          P~ = e2m1_rne(6 * 2^x')          (block scale 1),
       quantise-after-exp: p = 2^x', per 16 keys sf = ue4m3_rne(amax(p)/6),
                           P~ = e2m1_rne(p / sf) * sf;
     with p_unit = 6 (Direct-P) or 1, l and acc accumulate P~ / p_unit and
     (P~ . deq(V)) / p_unit.
  4. O = acc / l, LSE = ln2 * (m + log2 l).

Value sets of e2m1 and e4m3 are those of the OCP Microscaling Formats (MX)
v1.0 specification: e2m1 = {0, .5, 1, 1.5, 2, 3, 4, 6} (sign bit on top);
e4m3 = exponent bias 7, three mantissa bits, subnormals at exponent 0, largest
finite 448, 0x7F the NaN.
"""
from __future__ import annotations

import math

import numpy as np

from .attention import LN2, LOG2E, _f64, visible_mask
from .outcomes import FlipRecorder, OutcomeRange, eval_band, near_midpoint, subset_options

F32 = np.float32


# ----------------------------------------------------------------------------
# INT8
# ----------------------------------------------------------------------------

def quantize_int8_rows(x):
    """Symmetric INT8 with one fp32 scale per row (last axis = channels).

    s = amax / 127 in fp32; q = clamp(rne(x / s), -127, 127) with an IEEE fp32
    divide; amax == 0 gives s = 1 and q = 0.  Returns (q int8, s float32)."""
    xf = _f64(x).astype(F32)                    # bf16 -> fp32 is exact
    amax = np.abs(xf).max(axis=-1)
    s = (amax / F32(127.0)).astype(F32)
    s = np.where(amax == 0, F32(1.0), s).astype(F32)
    qf = np.rint((xf / s[..., None]).astype(F32))
    q = np.clip(qf, -127, 127).astype(np.int8)
    return q, s


def quantize_int4_rows(x):
    """Symmetric INT4 with one fp32 scale per row, the token-level scheme at 4
    bits ([INT-FA]: the token-level quantisation carries over to lower
    formats such as INT4): s = amax / 7 in fp32, q = clamp(rne(x / s), -7, 7)
    with an IEEE fp32 divide, amax == 0 gives s = 1 and q = 0.  The codes are
    returned in int8 containers (the INT8 forward consumes them unchanged).
    Returns (q int8 in [-7, 7], s float32)."""
    xf = _f64(x).astype(F32)
    amax = np.abs(xf).max(axis=-1)
    s = (amax / F32(7.0)).astype(F32)
    s = np.where(amax == 0, F32(1.0), s).astype(F32)
    qf = np.rint((xf / s[..., None]).astype(F32))
    q = np.clip(qf, -7, 7).astype(np.int8)
    return q, s


def quantize_int8_heads(x):
    """Symmetric INT8 with one fp32 scale per (batch, head) of a [B,H,N,d]
    tensor (the V operand).  Same formula as ``quantize_int8_rows``."""
    xf = _f64(x).astype(F32)
    amax = np.abs(xf).max(axis=(-2, -1))
    s = (amax / F32(127.0)).astype(F32)
    s = np.where(amax == 0, F32(1.0), s).astype(F32)
    qf = np.rint((xf / s[..., None, None]).astype(F32))
    q = np.clip(qf, -127, 127).astype(np.int8)
    return q, s


def int8_scores(qi, ki):
    """Exact integer Q K^T of INT8 operands: [B,H,Nq,Nkv] int32."""
    S = np.einsum("bhid,bhjd->bhij", qi.astype(np.int64), ki.astype(np.int64))
    assert np.abs(S).max(initial=0) < 2 ** 31
    return S.astype(np.int32)


def attention_int8(qi, qs, ki, ks, vi, vs, causal=False, scale=None, Bc=128,
                   outcomes=False, rows=None):
    """Emulated INT8 forward (steps 2-5 of the module docstring).

    qi, ki, vi: int8 [B,H,N,d]; qs, ks: fp32 [B,H,N]; vs: fp32 [B,H].
    ``rows`` restricts the computation to those query rows (rows are
    independent).  Returns (O, LSE) float64 and, with ``outcomes``, also an
    ``OutcomeRange``: the interval of O and LSE over both roundings of every
    element of 127 * 2^(x - m) that lies within fp32 evaluation error of a
    rounding midpoint (``oracle.outcomes``).
    """
    qi, ki, vi = np.asarray(qi), np.asarray(ki), np.asarray(vi)
    qs, ks, vs = _f64(qs), _f64(ks), _f64(vs)
    B, H, Nq_all, d = qi.shape
    Nkv = ki.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ridx = np.arange(Nq_all) if rows is None else np.asarray(rows, dtype=np.int64)
    Nq = ridx.size
    O = np.zeros((B, H, Nq, d))
    LSE = np.full((B, H, Nq), -np.inf)
    rng = _RangeCollector(O.shape) if outcomes else None
    grid = np.arange(128.0)
    vis = visible_mask(Nq_all, Nkv, causal, ridx)
    for b in range(B):
        for h in range(H):
            S = qi[b, h, ridx].astype(np.int64) @ ki[b, h].astype(np.int64).T
            x = S * (qs[b, h, ridx][:, None] * ks[b, h][None, :]) * (scale * LOG2E)
            x = np.where(vis, x, -np.inf)
            acc = np.zeros((Nq, d))
            l = np.zeros(Nq)
            m = np.full(Nq, -np.inf)
            rec = FlipRecorder()
            for j0 in range(0, Nkv, Bc):
                cols = slice(j0, min(Nkv, j0 + Bc))
                xb = x[:, cols]
                m_new = np.maximum(m, xb.max(axis=1))
                grow = np.isfinite(m) & (m_new > m)
                f = np.ones_like(m)
                with np.errstate(invalid="ignore"):  # -inf - -inf in lanes the where() discards
                    np.exp2(m - m_new, out=f, where=grow)
                acc *= f[:, None]
                l *= f
                m = m_new
                ms = np.where(np.isfinite(m), m, 0.0)
                fin = np.isfinite(xb) & np.isfinite(m)[:, None]
                p = np.zeros_like(xb)
                np.exp2(np.where(fin, xb - ms[:, None], 0.0), out=p, where=fin)
                y = 127.0 * p
                P8 = np.rint(y)
                if outcomes:
                    band = eval_band(y, np.where(fin, xb, 0.0), ms[:, None], 1e-12)
                    flag, alt = near_midpoint(y, grid, P8, band)
                    r_, c_ = np.nonzero(flag & fin)
                    rec.add_elements(r_, c_ + j0, (alt - P8)[r_, c_], ms[r_])
                l += P8.sum(axis=1) / 127.0
                acc += (P8 @ vi[b, h, cols].astype(np.float64)) * (vs[b, h] / 127.0)
            ok = l > 0
            ls = np.where(ok, l, 1.0)
            O[b, h] = np.where(ok[:, None], acc / ls[:, None], 0.0)
            LSE[b, h] = np.where(ok, LN2 * (np.where(ok, m, 0.0) + np.log2(ls)), -np.inf)
            if outcomes:
                U = vi[b, h].astype(np.float64) * (vs[b, h] / 127.0)
                rng.add(b, h, rec, acc, l, m, U, 1.0 / 127.0)
    if outcomes:
        return O, LSE, rng.result(O, LSE)
    return O, LSE


class _RangeCollector:
    """Gathers the per-(b, h) intervals of a blockwise quantised forward into
    one ``OutcomeRange``."""

    def __init__(self, shape):
        self.O_lo = np.zeros(shape)
        self.O_hi = np.zeros(shape)
        self.l_lo = np.zeros(shape[:-1])
        self.l_hi = np.zeros(shape[:-1])
        self.m = np.zeros(shape[:-1])
        self.flips = 0
        self.flagged_rows = 0
        self.ambiguous = 0

    def add(self, b, h, rec, num, l, m, U, w):
        lo, hi, llo, lhi = rec.intervals(num, l, m, U, w)
        self.O_lo[b, h], self.O_hi[b, h] = lo, hi
        self.l_lo[b, h], self.l_hi[b, h] = llo, lhi
        self.m[b, h] = np.where(np.isfinite(m), m, 0.0)
        self.flips += rec.count()
        self.flagged_rows += len(rec.vars)

    def widen(self, b, h, r, lo, hi, llo, lhi, m):
        """Hull of row r's interval with another decision path's, whose
        reference max is m (the LSE ends are compared on a common base)."""
        self.O_lo[b, h, r] = np.minimum(self.O_lo[b, h, r], lo)
        self.O_hi[b, h, r] = np.maximum(self.O_hi[b, h, r], hi)
        m0 = self.m[b, h, r]
        # l at reference m equals l * 2^(m - m0) at reference m0
        self.l_lo[b, h, r] = min(self.l_lo[b, h, r], llo * 2.0 ** (m - m0))
        self.l_hi[b, h, r] = max(self.l_hi[b, h, r], lhi * 2.0 ** (m - m0))

    def result(self, O, LSE):
        fin = np.isfinite(LSE)
        lse_lo = np.where(fin, LN2 * (self.m + np.log2(np.where(fin, self.l_lo, 1.0))), -np.inf)
        lse_hi = np.where(fin, LN2 * (self.m + np.log2(np.where(fin, self.l_hi, 1.0))), -np.inf)
        # rows that see no key: O = 0 exactly on both sides
        O_lo = np.where(fin[..., None], self.O_lo, O)
        O_hi = np.where(fin[..., None], self.O_hi, O)
        return OutcomeRange(O_lo, O_hi, lse_lo, lse_hi, self.flips, self.flagged_rows,
                            int(np.prod(LSE.shape)), self.ambiguous)


# ----------------------------------------------------------------------------
# FP4 (e2m1 codes with unsigned-e4m3 block scales, 16 elements per block)
# ----------------------------------------------------------------------------

E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(codes):
    """4-bit codes (sign in bit 3) -> float64 values."""
    c = np.asarray(codes).astype(np.int64)
    mag = E2M1_VALUES[c & 7]
    return np.where(c & 8, -mag, mag)


def e2m1_encode(x):
    """Round to nearest e2m1, ties to the even code, saturating at +-6.
    Brute force over the eight magnitudes.  NaN is not expected."""
    xf = _f64(x)
    a = np.minimum(np.abs(xf), 6.0)
    dist = np.abs(a[..., None] - E2M1_VALUES)                 # [..., 8]
    best = dist.min(axis=-1, keepdims=True)
    cand = dist == best
    # among equally near codes take the even one (codes are 0..7, ascending)
    even = cand & ((np.arange(8) % 2) == 0)
    code = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(cand, axis=-1))
    neg = np.signbit(xf) & (code != 0)
    return (code + 8 * neg).astype(np.uint8)


def _e4m3_table():
    vals = np.zeros(127)
    for c in range(127):          # 0x00 .. 0x7E are finite
        e, mnt = c >> 3, c & 7
        vals[c] = (mnt / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + mnt / 8.0) * 2.0 ** (e - 7)
    return vals


UE4M3_VALUES = _e4m3_table()


def ue4m3_decode(codes):
    """Unsigned e4m3 code (0x00..0x7E) -> float64."""
    return UE4M3_VALUES[np.asarray(codes).astype(np.int64)]


def ue4m3_encode(x):
    """Round a non-negative value to nearest unsigned e4m3, ties to the even
    code, saturating at 448."""
    a = np.minimum(_f64(x), 448.0)
    hi = np.searchsorted(UE4M3_VALUES, a, side="left")        # first value >= a
    hi = np.clip(hi, 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    dl = np.abs(a - UE4M3_VALUES[lo])
    dh = np.abs(UE4M3_VALUES[hi] - a)
    pick_hi = (dh < dl) | ((dh == dl) & (hi % 2 == 0))
    return np.where(pick_hi, hi, lo).astype(np.uint8)


def quantize_nvfp4(x, axis=-1, block=16):
    """NVFP4 quantisation with blocks of ``block`` along ``axis``.

    amax per block (fp32), sf = ue4m3_rne(amax / 6) (fp32 divide), codes =
    e2m1_rne_satfinite(x / deq(sf)) (fp32 divide); a zero scale gives zero
    codes.  Returns (codes uint8 [x.shape], sf uint8 [x.shape with axis/16])."""
    xf = np.moveaxis(_f64(x).astype(F32), axis, -1)
    n = xf.shape[-1]
    assert n % block == 0
    xb = xf.reshape(xf.shape[:-1] + (n // block, block))
    amax = np.abs(xb).max(axis=-1)
    sf = ue4m3_encode((amax / F32(6.0)).astype(F32))
    s = ue4m3_decode(sf).astype(F32)
    safe = np.where(s > 0, s, F32(1.0)).astype(F32)
    qv = (xb / safe[..., None]).astype(F32)
    codes = np.where((s > 0)[..., None], e2m1_encode(qv), 0).astype(np.uint8)
    codes = np.moveaxis(codes.reshape(xf.shape), -1, axis)
    sf = np.moveaxis(sf, -1, axis)
    return codes, sf


def nvfp4_dequantize(codes, sf, axis=-1, block=16):
    """deq = e2m1(code) * ue4m3(sf) with the scale broadcast over its block."""
    c = np.moveaxis(np.asarray(codes), axis, -1)
    s = np.moveaxis(np.asarray(sf), axis, -1)
    vals = e2m1_decode(c) * np.repeat(ue4m3_decode(s), block, axis=-1)
    return np.moveaxis(vals, -1, axis)


DIRECT_P, QUANT_AFTER_EXP = 0, 1


def direct_p_values(xp):
    """Direct-P: the e2m1 value nearest to 6 * 2^x' (x' = x - m <= 0), ties to
    the even code, as the P operand with a unit block scale.  [FP4-FA4]: the
    raw score is mapped straight to the FP4 code; no probability is formed and
    rescaled first.  Returns (values in [0, 6], codes)."""
    xp = _f64(xp)
    y = np.where(np.isfinite(xp), 6.0 * np.exp2(np.minimum(xp, 0.0)), 0.0)
    codes = e2m1_encode(y)
    return e2m1_decode(codes), codes


def quant_after_exp_values(p, block=16):
    """Quantise-after-exp: per 16 consecutive keys sf = ue4m3_rne(amax(p)/6) and
    e2m1_rne(p / sf).  ``p`` is [..., keys] (keys a multiple of 16) in [0, 1].
    Returns (dequantised values, codes, sf)."""
    codes, sf = quantize_nvfp4(p, axis=-1, block=block)
    return nvfp4_dequantize(codes, sf, axis=-1, block=block), codes, sf


def attention_fp4(q_deq, k_deq, v_deq, p_mode=DIRECT_P, causal=False, scale=None,
                  Bc=128, outcomes=False):
    """Emulated FP4 forward (steps 2-4 of the module docstring).

    q_deq, k_deq, v_deq: dequantised NVFP4 operands [B,H,N,d] (float64; use
    ``nvfp4_dequantize``).  Returns (O, LSE) and, with ``outcomes``, also an
    ``OutcomeRange`` over both roundings of every P element that lies within
    the device's fp32 evaluation error of an e2m1 rounding midpoint, and, for
    quantise-after-exp, over both roundings of a block scale amax / 6 that
    lies that close to an e4m3 midpoint (the block's codes then follow the
    chosen scale).  See ``oracle.outcomes``."""
    q, k, v = _f64(q_deq), _f64(k_deq), _f64(v_deq)
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    p_unit = 6.0 if p_mode == DIRECT_P else 1.0
    O = np.zeros((B, H, Nq, d))
    LSE = np.full((B, H, Nq), -np.inf)
    rng = _RangeCollector(O.shape) if outcomes else None
    vis = visible_mask(Nq, Nkv, causal)
    for b in range(B):
        for h in range(H):
            x = (q[b, h] @ k[b, h].T) * (scale * LOG2E)
            x = np.where(vis, x, -np.inf)
            acc = np.zeros((Nq, d))
            l = np.zeros(Nq)
            m = np.full(Nq, -np.inf)
            rec = FlipRecorder()
            for j0 in range(0, Nkv, Bc):
                j1 = min(Nkv, j0 + Bc)
                cols = slice(j0, j1)
                xb = x[:, cols]
                m_new = np.maximum(m, xb.max(axis=1))
                grow = np.isfinite(m) & (m_new > m)
                f = np.ones_like(m)
                with np.errstate(invalid="ignore"):  # -inf - -inf in lanes the where() discards
                    np.exp2(m - m_new, out=f, where=grow)
                acc *= f[:, None]
                l *= f
                m = m_new
                ms = np.where(np.isfinite(m), m, 0.0)
                fin = np.isfinite(xb) & np.isfinite(m)[:, None]
                xp = np.where(fin, xb - ms[:, None], -np.inf)
                if p_mode == DIRECT_P:
                    Pt, _ = direct_p_values(xp)
                    if outcomes:
                        y = np.where(fin, 6.0 * np.exp2(np.minimum(np.where(fin, xp, 0.0), 0.0)), 0.0)
                        band = eval_band(y, np.where(fin, xb, 0.0), ms[:, None], 1e-12)
                        flag, alt = near_midpoint(y, E2M1_VALUES, Pt, band)
                        r_, c_ = np.nonzero(flag & fin)
                        rec.add_elements(r_, c_ + j0, (alt - Pt)[r_, c_], ms[r_])
                else:
                    width = j1 - j0
                    pad = (-width) % 16
                    p = np.zeros_like(xb)
                    np.exp2(np.where(fin, xp, 0.0), out=p, where=fin)
                    p32 = p.astype(F32)
                    pp = np.pad(p32, ((0, 0), (0, pad)))
                    Pt_full, _, sf = quant_after_exp_values(pp)
                    Pt = Pt_full[:, :width]
                    if outcomes:
                        xe = np.pad(np.where(fin, xb, 0.0), ((0, 0), (0, pad)))
                        _qae_flips(rec, pp.astype(np.float64), Pt_full, sf, xe, ms, j0, width)
                l += Pt.sum(axis=1) / p_unit
                acc += (Pt @ v[b, h, cols]) / p_unit
            ok = l > 0
            ls = np.where(ok, l, 1.0)
            O[b, h] = np.where(ok[:, None], acc / ls[:, None], 0.0)
            LSE[b, h] = np.where(ok, LN2 * (np.where(ok, m, 0.0) + np.log2(ls)), -np.inf)
            if outcomes:
                rng.add(b, h, rec, acc, l, m, v[b, h] / p_unit, 1.0 / p_unit)
    if outcomes:
        return O, LSE, rng.result(O, LSE)
    return O, LSE


def _qae_codes(p, s):
    """Rows of 16 fp32 probabilities p [R, 16] against scales s [R]: the ratio
    p / s (fp32 divide, zero where s = 0), its e2m1 magnitude and the
    dequantised value (magnitude * s)."""
    s32 = np.asarray(s, dtype=F32)
    safe = np.where(s32 > 0, s32, F32(1.0)).astype(F32)
    r = np.where((s32 > 0)[:, None], (p.astype(F32) / safe[:, None]).astype(F32), F32(0.0)).astype(np.float64)
    mag = np.abs(e2m1_decode(e2m1_encode(r)))
    return mag * np.asarray(s, dtype=np.float64)[:, None], r, mag


def _qae_flips(rec, pp, Pt_full, sf, xe, ms, j0, width):
    """Flagged variables of one key block under quantise-after-exp.

    pp [R, n16] the block's fp32 probabilities (zero padded to 16-key groups),
    Pt_full their oracle values, sf the oracle's e4m3 scale codes [R, n16/16],
    xe the scores (0 where masked or padded), ms the row reference max.  A
    16-key group whose amax / 6 lies within evaluation error of an e4m3
    midpoint becomes one variable whose options are the other scale's codes
    and every admissible rounding of the codes under either scale; otherwise
    each code whose p / sf lies near an e2m1 midpoint is one binary variable."""
    R, n = pp.shape
    s_all = ue4m3_decode(sf)                               # [R, n/16]
    for g in range(n // 16):
        c0, c1 = g * 16, min(width, g * 16 + 16)
        if c1 <= c0:
            continue
        nkeep = c1 - c0
        p = pp[:, c0:c0 + 16]
        xg = xe[:, c0:c0 + 16]
        base = Pt_full[:, c0:c0 + 16]
        s = s_all[:, g]
        a = (p.max(axis=1).astype(F32) / F32(6.0)).astype(np.float64)
        sflag, s_alt = near_midpoint(a, UE4M3_VALUES, s, eval_band(a, np.abs(xg).max(axis=1), ms, 1e-12))
        _, ratio, mag = _qae_codes(p, s)
        cflag, calt = near_midpoint(ratio, E2M1_VALUES, mag, eval_band(ratio, xg, ms[:, None], 1e-12))
        cflag &= p > 0
        keys = np.arange(j0 + c0, j0 + c1)
        for r in np.flatnonzero(sflag | cflag[:, :nkeep].any(axis=1)):
            s_r = s[r]
            if sflag[r]:
                opts = []
                if cflag[r].any():
                    opts.append(subset_options(base[r], calt[r] * s_r, cflag[r]))
                va, ra, ma = _qae_codes(p[r:r + 1], s_alt[r:r + 1])
                aflag, aalt = near_midpoint(ra[0], E2M1_VALUES, ma[0], eval_band(ra[0], xg[r], ms[r], 1e-12))
                aflag &= p[r] > 0
                opts.append((va[0] - base[r])[None, :])
                if aflag.any():
                    opts.append(subset_options(va[0], aalt * s_alt[r], aflag) + (va[0] - base[r])[None, :])
                rec.add_group(r, keys, np.vstack(opts)[:, :nkeep], ms[r])
            else:
                js = np.flatnonzero(cflag[r, :nkeep])
                rec.add_elements(np.full(js.size, r), keys[js], (calt[r] * s_r - base[r])[js],
                                 np.full(js.size, ms[r]))
