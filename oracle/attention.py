"""fp64 reference for scaled-dot-product attention (bf16 path and decode).

TEST INFRASTRUCTURE ONLY (see the package docstring): the tests, the smoke
check and the benchmark's CPU baseline call this; the product never does.

Everything is float64 numpy.  Inputs may be any real dtype; bf16 tensors are
converted exactly (every bf16 value is a float64 value).  Shapes are
[B][H][N][d] as in [FA-trading] "Integration in eight lines" (q, k, v shaped
(batch, heads, seq, head_dim)).

Causal alignment (the pages only say "the model must not look at the future",
[FA-trading] "Causal masking"): key j is visible to query i iff
j <= i + (Nkv - Nq), i.e. the last query sees every key.  For Nq == Nkv this is
the usual lower-triangular mask of the explicit-score code in "Integration in
eight lines".  A query row that sees no key gets O = 0 and LSE = -inf.

LSE is the natural-log log-sum-exp of the scaled scores,
LSE_i = log sum_j exp(scale * q_i . k_j): the per-row softmax statistics that
[FA-trading] "Backward: recompute instead of store" keeps instead of P.
"""
from __future__ import annotations

import math

import numpy as np

from .outcomes import near_midpoint

LOG2E = 1.0 / math.log(2.0)
LN2 = math.log(2.0)


def _f64(x) -> np.ndarray:
    """Exact conversion of a numpy array or a torch tensor to float64 numpy."""
    if hasattr(x, "detach"):  # torch tensor, any dtype; .double() is exact
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def visible_mask(Nq: int, Nkv: int, causal: bool, rows=None) -> np.ndarray:
    """Boolean [rows][Nkv]: True where key j is visible to query i."""
    i = np.arange(Nq) if rows is None else np.asarray(rows)
    j = np.arange(Nkv)
    if not causal:
        return np.ones((i.size, Nkv), dtype=bool)
    return j[None, :] <= (i[:, None] + (Nkv - Nq))


def attention(q, k, v, causal: bool = False, scale: float | None = None,
              rows=None, row_chunk: int = 1024):
    """O = softmax(scale * Q K^T, masked) V and LSE, the plain definition.

    [FA-trading] "Why attention is memory-bound": softmax(Q K^T / sqrt(d_k)) V,
    with the N x N score matrix S = Q K^T / sqrt(d_k) materialised;
    "Integration in eight lines": scores, masked_fill(-inf), softmax, matmul.

    ``rows`` optionally restricts the computation to a subset of query rows
    (same rows for every (b, h)); the result then has len(rows) query rows.
    Rows are processed ``row_chunk`` at a time (rows are independent, so this is
    the same definition, only with less memory).

    Returns (O [B,H,R,d] float64, LSE [B,H,R] float64).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    row_idx = np.arange(Nq) if rows is None else np.asarray(rows, dtype=np.int64)
    R = row_idx.size
    O = np.zeros((B, H, R, v.shape[3]), dtype=np.float64)
    LSE = np.full((B, H, R), -np.inf, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for r0 in range(0, R, row_chunk):
                ri = row_idx[r0:r0 + row_chunk]
                S = (q[b, h, ri] @ k[b, h].T) * scale           # [r, Nkv]
                S = np.where(visible_mask(Nq, Nkv, causal, ri), S, -np.inf)
                m = S.max(axis=1)
                alive = np.isfinite(m)
                m_safe = np.where(alive, m, 0.0)
                P = np.exp(S - m_safe[:, None])                  # exp(-inf) = 0
                l = P.sum(axis=1)
                l_safe = np.where(alive, l, 1.0)
                P = P / l_safe[:, None]
                O[b, h, r0:r0 + ri.size] = np.where(alive[:, None], P @ v[b, h], 0.0)
                LSE[b, h, r0:r0 + ri.size] = np.where(alive, m_safe + np.log(l_safe),
                                                       -np.inf)
    return O, LSE


def attention_backward(q, k, v, do, causal: bool = False, scale: float | None = None, p_round=None,
                       p_grid=None, p_rel=2e-5):
    """Gradients of O = softmax(scale * Q K^T, masked) V with respect to Q, K
    and V for an upstream gradient dO, in float64 -- the calculus of the
    definition, with P materialised (the quantity [FA-trading] "Backward:
    recompute instead of store" says the tiled method recomputes from Q, K and
    the stored softmax statistics instead of keeping it):

        dV = P^T dO,  dP = dO V^T,  dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik),
        dQ = scale dS K,  dK = scale dS^T Q.

    sum_k P_ik dP_ik equals sum_c dO_ic O_ic (O = P V).  Rows that see no key
    have P = 0 and contribute nothing.  Returns (dQ, dK, dV) float64.

    ``p_round`` (a function on arrays) rounds P where it is the operand of
    dV = round(P)^T dO only (the FP8-P backward of [FP4-FA4]: 8-bit
    probabilities in the backward); dS keeps P unrounded.  With ``p_grid``
    (the sorted non-negative values ``p_round`` rounds to) it also returns
    the interval (dV_lo, dV_hi) of dV over both roundings of every P element
    within ``p_rel`` (relative) of a rounding midpoint of that grid: dV is
    linear in the rounded P, so each such element adds its change times dO
    to one end of the interval (``oracle.outcomes``)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dv_lo = np.zeros_like(v)
    dv_hi = np.zeros_like(v)
    vis = visible_mask(Nq, Nkv, causal)
    for b in range(B):
        for h in range(H):
            S = np.where(vis, (q[b, h] @ k[b, h].T) * scale, -np.inf)
            m = S.max(axis=1)
            alive = np.isfinite(m)
            P = np.exp(S - np.where(alive, m, 0.0)[:, None])
            P /= np.where(alive, P.sum(axis=1), 1.0)[:, None]
            P = np.where(alive[:, None], P, 0.0)
            dP = do[b, h] @ v[b, h].T
            dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            Pv = P if p_round is None else p_round(P)
            dv[b, h] = Pv.T @ do[b, h]
            dq[b, h] = scale * (dS @ k[b, h])
            dk[b, h] = scale * (dS.T @ q[b, h])
            if p_grid is not None:
                flag, alt = near_midpoint(P, p_grid, Pv, p_rel * P)
                delta = np.where(flag & (P > 0), alt - Pv, 0.0)             # [Nq, Nkv]
                up, dn = np.maximum(delta, 0.0), np.minimum(delta, 0.0)
                dpos, dneg = np.maximum(do[b, h], 0.0), np.minimum(do[b, h], 0.0)
                # sum_i min(0, delta_ij dO_ic) and sum_i max(0, delta_ij dO_ic)
                dv_lo[b, h] = dv[b, h] + up.T @ dneg + dn.T @ dpos
                dv_hi[b, h] = dv[b, h] + up.T @ dpos + dn.T @ dneg
    if p_grid is not None:
        return dq, dk, dv, (dv_lo, dv_hi)
    return dq, dk, dv


def kv_head_index(Hq: int, Hkv: int) -> np.ndarray:
    """Key/value head of every query head under grouped-query attention:
    query head h reads key/value head h // (Hq / Hkv) ([FA4-overview]
    "Compatibility and current status": several attention heads share one
    key/value projection; Hkv = 1 is multi-query attention, Hkv = Hq plain
    multi-head attention)."""
    if Hkv < 1 or Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return np.arange(Hq) // (Hq // Hkv)


def attention_gqa(q, k, v, causal: bool = False, scale: float | None = None, rows=None):
    """Grouped-query attention: the plain definition with each query head's
    key/value head substituted (q [B,Hq,Nq,d], k/v [B,Hkv,Nkv,d])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    idx = kv_head_index(q.shape[1], k.shape[1])
    return attention(q, k[:, idx], v[:, idx], causal, scale, rows=rows)


def softmax_rows(q, k, causal: bool = False, scale: float | None = None):
    """The normalised probability matrix P [B,H,Nq,Nkv] (small inputs only)."""
    q, k = _f64(q), _f64(k)
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    S = np.einsum("bhid,bhjd->bhij", q, k) * scale
    S = np.where(visible_mask(Nq, Nkv, causal)[None, None], S, -np.inf)
    m = S.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    P = np.exp(S - m)
    l = P.sum(axis=-1, keepdims=True)
    return P / np.where(l > 0, l, 1.0)


def _exp_shift(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """exp(a - b) with the convention exp(-inf - (-inf)) = 0 (nothing seen yet)."""
    out = np.zeros(np.broadcast(a, b).shape)
    ok = np.isfinite(a) & np.isfinite(b)
    np.exp(np.where(ok, a - np.where(np.isfinite(b), b, 0.0), 0.0), out=out, where=ok)
    return out


def attention_blockwise(q, k, v, causal: bool = False, scale: float | None = None,
                        Br: int = 128, Bc: int = 128):
    """The tiled forward as [FA-trading] "The Flash Attention algorithm" states
    it: Q in T_r = ceil(N/B_r) row blocks, K/V in T_c = ceil(N/B_c) column
    blocks; per KV block a local row max m_ij, P_ij = exp(S_ij - m_ij), local
    sum l_ij, then the running (m, l) and the normalised output O_i updated with
    the factors l_i e^{m_i - m_new} / l_new and e^{m_ij - m_new} / l_new.

    A second, independent route to the same numbers as ``attention``; used by
    the oracle's self-tests.  Returns (O, LSE) with LSE = m + log l.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.zeros((B, H, Nq, v.shape[3]))
    LSE = np.full((B, H, Nq), -np.inf)
    for b in range(B):
        for h in range(H):
            for i0 in range(0, Nq, Br):
                rows = np.arange(i0, min(Nq, i0 + Br))
                Oi = np.zeros((rows.size, v.shape[3]))
                mi = np.full(rows.size, -np.inf)
                li = np.zeros(rows.size)
                vis = visible_mask(Nq, Nkv, causal, rows)
                for j0 in range(0, Nkv, Bc):
                    cols = slice(j0, min(Nkv, j0 + Bc))
                    Sij = (q[b, h, rows] @ k[b, h, cols].T) * scale
                    Sij = np.where(vis[:, cols], Sij, -np.inf)
                    mij = Sij.max(axis=1)
                    Pij = _exp_shift(Sij, mij[:, None])
                    lij = Pij.sum(axis=1)
                    m_new = np.maximum(mi, mij)
                    a_old = li * _exp_shift(mi, m_new)
                    a_new = _exp_shift(mij, m_new)
                    l_new = a_old + lij * a_new
                    ok = l_new > 0
                    inv = np.where(ok, 1.0 / np.where(ok, l_new, 1.0), 0.0)
                    Oi = Oi * (a_old * inv)[:, None] + (Pij @ v[b, h, cols]) * (a_new * inv)[:, None]
                    mi, li = m_new, l_new
                O[b, h, rows] = Oi
                LSE[b, h, rows] = np.where(li > 0, mi + np.log(np.where(li > 0, li, 1.0)),
                                           -np.inf)
    return O, LSE


def attention_lazy_rescale(q, k, v, causal: bool = False, scale: float | None = None,
                           Bc: int = 128, tau: float = 8.0, count_rescales: bool = False,
                           rescale_rows: bool = False):
    """The deferred-normalisation form with lazy rescaling, base 2.

    [FA-trading] "FA2" item 1: the output accumulator stays unnormalised and is
    divided by l once after the inner loop.  [FA4-overview] "Smarter online
    softmax rescaling": the reference maximum only moves (and O, l are only
    rescaled) when the new block maximum exceeds it by a significant amount;
    the pages give no constant, ``tau`` is that amount in log2 units (tau = 0
    rescales on every increase, the classic recurrence of "Online softmax
    recurrence").  Scores are handled as base-2 logits x = scale * S * log2(e)
    ([FA4-overview] "Software exponent on CUDA cores": the kernel evaluates
    exp2).  Exact in exact arithmetic for every tau, because O and l share the
    same stale reference.

    Returns (O, LSE) and, if ``count_rescales``, the number of (row, block)
    pairs in which the reference moved after the first block.  With
    ``rescale_rows`` it returns (O, LSE, moves, margin) instead: per query row
    ([B, H, Nq]) the number of such moves, and the smallest distance
    |m_blk - (m + tau)| of any of its decisions after the first block (inf for
    a row with none) -- how close the row came to the threshold.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.zeros((B, H, Nq, v.shape[3]))
    LSE = np.full((B, H, Nq), -np.inf)
    vis = visible_mask(Nq, Nkv, causal)
    rescales = 0
    moves = np.zeros((B, H, Nq), dtype=np.int64)
    margin = np.full((B, H, Nq), np.inf)
    for b in range(B):
        for h in range(H):
            acc = np.zeros((Nq, v.shape[3]))
            l = np.zeros(Nq)
            m = np.full(Nq, -np.inf)
            for jb, j0 in enumerate(range(0, Nkv, Bc)):
                cols = slice(j0, min(Nkv, j0 + Bc))
                x = (q[b, h] @ k[b, h, cols].T) * (scale * LOG2E)
                x = np.where(vis[:, cols], x, -np.inf)
                m_blk = x.max(axis=1)
                m_new = np.maximum(m, m_blk)
                move = np.isfinite(m_new) & (~np.isfinite(m) | (m_new > m + tau))
                if jb > 0:
                    rescales += int(np.count_nonzero(move & np.isfinite(m)))
                    moves[b, h] += move & np.isfinite(m)
                    decided = np.isfinite(m) & np.isfinite(m_blk)
                    with np.errstate(invalid="ignore"):
                        gap = np.abs(m_blk - (m + tau))
                    margin[b, h] = np.where(decided, np.minimum(margin[b, h], gap), margin[b, h])
                with np.errstate(invalid="ignore"):  # -inf - -inf in lanes the where() discards
                    f = np.where(move & np.isfinite(m),
                                 np.exp2(np.where(move & np.isfinite(m), m - m_new, 0.0)), 1.0)
                acc *= f[:, None]
                l *= f
                m = np.where(move, m_new, m)
                p = np.zeros_like(x)
                fin = np.isfinite(x) & np.isfinite(m)[:, None]
                np.exp2(np.where(fin, x - np.where(np.isfinite(m), m, 0.0)[:, None], 0.0),
                        out=p, where=fin)
                l += p.sum(axis=1)
                acc += p @ v[b, h, cols]
            ok = l > 0
            ls = np.where(ok, l, 1.0)
            O[b, h] = np.where(ok[:, None], acc / ls[:, None], 0.0)
            LSE[b, h] = np.where(ok, LN2 * (np.where(ok, m, 0.0) + np.log2(ls)), -np.inf)
    if rescale_rows:
        return O, LSE, moves, margin
    if count_rescales:
        return O, LSE, rescales
    return O, LSE


def split_bounds(Nkv: int, num_splits: int):
    """Key ranges of a split-KV decode: equal chunks of ceil(Nkv / splits) keys
    (the last ones may be short or empty)."""
    chunk = -(-Nkv // num_splits)
    return [(min(Nkv, c * chunk), min(Nkv, (c + 1) * chunk)) for c in range(num_splits)]


def decode_partials(q, k, v, scale: float | None = None, num_splits: int = 16):
    """Per split c: attention of the query rows over keys of chunk c alone,
    giving (O_c, LSE_c).  An empty chunk gives O_c = 0, LSE_c = -inf.

    Returns (O_parts [S,B,H,Nq,d], LSE_parts [S,B,H,Nq])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    Os, Ls = [], []
    for lo, hi in split_bounds(k.shape[2], num_splits):
        if hi <= lo:
            Os.append(np.zeros((B, H, Nq, v.shape[3])))
            Ls.append(np.full((B, H, Nq), -np.inf))
            continue
        o, lse = attention(q, k[:, :, lo:hi], v[:, :, lo:hi], False, scale)
        Os.append(o)
        Ls.append(lse)
    return np.stack(Os), np.stack(Ls)


def combine(O_parts, LSE_parts):
    """LSE-weighted merge of split results: LSE = log sum_c exp(LSE_c) and
    O = sum_c exp(LSE_c - LSE) O_c.  The same identity as the online-softmax
    recurrence ([FA-trading] "Online softmax recurrence"), applied once to
    whole chunks instead of tile by tile."""
    O_parts, LSE_parts = _f64(O_parts), _f64(LSE_parts)
    mx = LSE_parts.max(axis=0)
    alive = np.isfinite(mx)
    mxs = np.where(alive, mx, 0.0)
    w = _exp_shift(LSE_parts, mxs[None])
    tot = w.sum(axis=0)
    tots = np.where(alive, tot, 1.0)
    O = np.where(alive[..., None], (w[..., None] * O_parts).sum(axis=0) / tots[..., None], 0.0)
    LSE = np.where(alive, mxs + np.log(tots), -np.inf)
    return O, LSE


def decode(q, k, v, scale: float | None = None):
    """Decode reference: one (or a few) query rows against the whole cache,
    which is the plain definition (non-causal over all cached keys)."""
    return attention(q, k, v, causal=False, scale=scale)


def attention_varlen(q, k, v, cu_q, cu_k, causal: bool = False, scale: float | None = None):
    """Variable-length batch packed without padding ([FA4-overview]
    "Compatibility and current status": variable-length sequences): q
    [total_q][Hq][d], k/v [total_k][Hkv][d] token-major; sequence b owns rows
    [cu_q[b], cu_q[b+1]) and keys [cu_k[b], cu_k[b+1]) and is the plain
    definition on its own rows and keys (causal alignment per sequence).
    Returns O [total_q][Hq][d] (rows outside every sequence are 0) and LSE
    [Hq][total_q] (-inf there)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu_q, cu_k = np.asarray(cu_q, dtype=np.int64), np.asarray(cu_k, dtype=np.int64)
    total_q, Hq, d = q.shape
    O = np.zeros((total_q, Hq, v.shape[2]))
    LSE = np.full((Hq, total_q), -np.inf)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        if q1 <= q0:
            continue
        qb = q[q0:q1].transpose(1, 0, 2)[None]          # [1][Hq][n][d]
        if k1 <= k0:
            LSE[:, q0:q1] = -np.inf                       # no key: O = 0
            continue
        kb = k[k0:k1].transpose(1, 0, 2)[None]
        vb = v[k0:k1].transpose(1, 0, 2)[None]
        Ob, Lb = attention_gqa(qb, kb, vb, causal, scale)
        O[q0:q1] = Ob[0].transpose(1, 0, 2)
        LSE[:, q0:q1] = Lb[0]
    return O, LSE


def decode_varlen(q, k, v, seqlens, scale: float | None = None):
    """Decode with a cache length per batch entry: entry b attends to keys
    [0, seqlens[b]) of k/v [B][Hkv][Nmax][d] (grouped-query when Hkv < Hq);
    an entry with no keys gets O = 0, LSE = -inf."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, d = q.shape
    O = np.zeros((B, Hq, Nq, v.shape[3]))
    LSE = np.full((B, Hq, Nq), -np.inf)
    for b in range(B):
        n = int(seqlens[b])
        if n <= 0:
            continue
        Ob, Lb = attention_gqa(q[b:b + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n], False, scale)
        O[b], LSE[b] = Ob[0], Lb[0]
    return O, LSE
