// INT8 tiled attention forward for sm_100a (TMA + tcgen05 kind::i8 + TMEM).
//
// "INT-FlashAttention" page: Q, K and V quantised to INT8 with token-level
// scales, and the two matmuls of the FlashAttention forward run as INT8 GEMMs
// with int32 accumulation.  Steps per 128-key block j (same tiling, masking
// and online softmax as the bf16 kernel, "Can a full-day context beat one
// minute? ..." sections "The Flash Attention algorithm" and "Online softmax
// recurrence"):
//   S_j  = Q_i8 K_j,i8^T                         int32, exact (tensor core)
//   x    = S_j * s_Q[row] * s_K[key] * scale * log2(e)          fp32
//   m    = running row max, moved on EVERY increase (P must stay <= 1)
//   P8   = rne(127 * 2^(x - m)) in [0, 127]    int8, written to TMEM
//   ACC += P8 V_j,i8                             int32 (tensor core)
//   l    = l * 2^(m_old - m) + sum(P8) / 127
// When the max of a row moves, the int32 accumulator cannot be rescaled in
// place, so the row's ACC is folded into an fp32 accumulator OF
// (OF = (OF + ACC * s_V / 127) * 2^(m_old - m_new), ACC = 0).  At the end
// O = (OF + ACC * s_V / 127) / l (fp32 output) and LSE = ln2 * (m + log2 l).
//
// CTA = one (batch, head) x one 128-row query tile.  Warps: 0 TMA producer,
// 1 MMA issuer, then NPART groups of four softmax/fold/epilogue warps: TMEM
// lane quarter q is read by NPART warps, group g taking key columns
// [CW g, CW g + CW) of every block (CW = 128 / NPART) and output columns
// [CW g, CW g + CW) of O; the NPART threads of a row exchange their partial
// row max once per block through tagged shared-memory slots (xchg_put/get).
// NPART softmax warps per SM sub-partition give the scheduler NPART
// instruction streams while each waits on its dependency chain.
// TMEM: S_0 cols [0,128), S_1 [128,256) (double-buffered scores, so S_{j+1}
// is computed while block j is in the softmax), ACC [256,384) int32,
// OF [384,512) fp32.  P8_j lives inside S_{j%2}: keys [CW g, CW g + CW) in
// columns [CW g, CW g + CW / 4), so each group writes only columns it has
// itself read.
// Shared memory: Q tile (128 x 128 int8 = 16 KB) and a ring of K/V tiles,
// 128-byte swizzled.  d = 128 only.
#pragma once
#include "ptx.cuh"
#include "fwd_bf16.cuh"  // fwd_tile_kv_count, wait_bar_drain

namespace ta {

struct FwdI8Params {
  const float* q_scale;  // [BH][Nq]
  const float* k_scale;  // [BH][Nkv]
  const float* v_scale;  // [BH]
  float* o;              // [BH][Nq][128] fp32
  float* lse;            // [BH][Nq]
  int* s_out;            // optional [BH][Nq][Nkv] int32 scores (debug export), else null
  int Nq, Nkv, n_qt, Tc;
  int causal;
  int ks_vec;  // k_scale rows are 16-byte aligned (Nkv % 4 == 0): vector loads
  float sl2;
  unsigned long long timeout_ns;
};

// kind::i8 instruction descriptor: D = s32 (2), A = B = signed 8-bit (1),
// M = 128; b_mn: B stored MN-major.
__host__ __device__ constexpr uint32_t idesc_i8(int N, bool b_mn) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

// softmax warps per TMEM lane quarter: each takes CW = 128 / I8_PARTS key
// columns of a block (and the same number of output columns of O)
#ifndef TA_I8_PARTS
#define TA_I8_PARTS 2
#endif
struct FwdI8Cfg {
  static constexpr int D = 128;
  static constexpr int TILE = 128 * 128;  // bytes of a 128 x 128 int8 tile
  static constexpr int NSLOT = 8;
  static constexpr int NPART = TA_I8_PARTS, CW = 128 / NPART, NCH = CW / 32;  // parts, columns, 32-col chunks
  static constexpr int NSW = 4 * NPART;                                     // softmax warps
  static constexpr int Q_OFF = 0;
  static constexpr int SLOT_OFF = TILE;
  static constexpr int KC_OFF = SLOT_OFF + NSLOT * TILE;                    // [NSW warps][2 bufs][CW] floats
  static constexpr int XCH_OFF = KC_OFF + NSW * 2 * CW * 4;                 // [3 slots][NPART][128 rows] u64
  static constexpr int BAR_OFF = XCH_OFF + 3 * NPART * 128 * 8;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
  static constexpr int THREADS = 64 + 32 * NSW;
  static_assert(NPART == 2 || NPART == 4, "two or four softmax warps per lane quarter");
  static constexpr uint32_t ID_S = idesc_i8(128, false);
  static constexpr uint32_t ID_PV = idesc_i8(128, true);  // V is MN-major
};

struct FwdI8Bars {
  uint64_t q_full;
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint64_t s_full[2];
  uint64_t p_full[2];  // per block parity: block j + 1 can be released before the MMA thread saw block j
  uint64_t pv_done;
  uint64_t o_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(FwdI8Bars) <= 256, "barrier block too large");

__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// exact int32 -> fp32 for |v| < 2^22 (|S| <= 127 * 127 * 128 < 2^21)
__device__ __forceinline__ float i2f_small(uint32_t v) {
  return __int_as_float((int)v + 0x4B400000) - 12582912.f;
}

template <bool SCORES_ONLY>
__global__ void __launch_bounds__(FwdI8Cfg::THREADS, 1)
    fwd_int8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdI8Params p) {
  using C = FwdI8Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FwdI8Bars* bars = reinterpret_cast<FwdI8Bars*>(smem + C::BAR_OFF);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int BH = gridDim.x / p.n_qt;
  const int bh = p.causal ? (int)(blockIdx.x % BH) : (int)(blockIdx.x / p.n_qt);
  const int qt = p.causal ? p.n_qt - 1 - (int)(blockIdx.x / BH) : (int)(blockIdx.x % p.n_qt);
  const int r0 = qt * 128;
  const int n = fwd_tile_kv_count(r0, p.Nq, p.Nkv, p.Tc, p.causal);
  volatile int* abort_flag = &bars->abort;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(smem_u32(&bars->kv_full[s]), 1);
      mbar_init(smem_u32(&bars->kv_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->s_full[0]), 1);
    mbar_init(smem_u32(&bars->s_full[1]), 1);
    mbar_init(smem_u32(&bars->p_full[0]), 32 * C::NSW);
    mbar_init(smem_u32(&bars->p_full[1]), 32 * C::NSW);
    mbar_init(smem_u32(&bars->pv_done), 1);
    mbar_init(smem_u32(&bars->o_full), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  {
    // exchange slots start with tag 0 (no block uses it), whatever a previous CTA left
    unsigned long long* xz = reinterpret_cast<unsigned long long*>(smem + C::XCH_OFF);
    for (int i = threadIdx.x; i < 3 * C::NPART * 128; i += C::THREADS) xz[i] = 0ull;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;
  // load order: K_0, V_0, K_1, V_1, ... (scores-only: K_0, K_1, ...)
  auto kidx = [&](int j) { return SCORES_ONLY ? j : 2 * j; };
  auto vidx = [&](int j) { return 2 * j + 1; };

  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      if (!SCORES_ONLY) prefetch_tmap(&tmV);
      const uint32_t qbar = smem_u32(&bars->q_full);
      mbar_arrive_expect_tx(qbar, C::TILE);
      tma_load_3d(sbase + C::Q_OFF, &tmQ, qbar, 0, r0, bh);
      int it = 0;
      bool ok = true;
      for (int j = 0; j < n && ok; ++j) {
        for (int w = 0; w < (SCORES_ONLY ? 1 : 2) && ok; ++w, ++it) {
          const int slot = it % C::NSLOT;
          const uint32_t ph = (it / C::NSLOT) & 1;
          ok = wait_bar(smem_u32(&bars->kv_empty[slot]), ph ^ 1, abort_flag, p.timeout_ns);
          if (!ok) break;
          const uint32_t fb = smem_u32(&bars->kv_full[slot]);
          mbar_arrive_expect_tx(fb, C::TILE);
          tma_load_3d(sbase + C::SLOT_OFF + slot * C::TILE, w == 0 ? &tmK : &tmV, fb, 0, j * 128, bh);
        }
      }
      if (!ok) {
        wait_bar_drain(qbar, 0, p.timeout_ns);
        for (int back = 1; back <= C::NSLOT && it - back >= 0; ++back) {
          const int i2 = it - back;
          wait_bar_drain(smem_u32(&bars->kv_full[i2 % C::NSLOT]), (i2 / C::NSLOT) & 1, p.timeout_ns);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      bool ok = wait_bar(smem_u32(&bars->q_full), 0, abort_flag, p.timeout_ns);
      tc_fence_after();
      const uint64_t dQ = smem_desc(sbase + C::Q_OFF, 16, 1024);
      const uint64_t dK0 = smem_desc(sbase + C::SLOT_OFF, 16, 1024);
      const uint64_t dV0 = smem_desc(sbase + C::SLOT_OFF, C::TILE, 1024);
      auto issue_S = [&](int j) -> bool {
        const int it = kidx(j), s = it % C::NSLOT;
        if (!wait_bar(smem_u32(&bars->kv_full[s]), (it / C::NSLOT) & 1, abort_flag, p.timeout_ns)) return false;
        tc_fence_after();
        const uint64_t dk = dK0 + (uint64_t)(s * (C::TILE >> 4));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = 32 int8 per MMA
          mma_i8_ss(tbase + (j & 1) * 128, dQ + (uint64_t)(kk * 2), dk + (uint64_t)(kk * 2), C::ID_S, kk > 0);
        tc_commit(smem_u32(&bars->s_full[j & 1]));
        tc_commit(smem_u32(&bars->kv_empty[s]));
        return true;
      };
      if (ok && n == 0) tc_commit(smem_u32(&bars->o_full));
      if (ok && n > 0) ok = issue_S(0);
      if (ok && n > 1) ok = issue_S(1);
      for (int j = 0; j < n && ok && !SCORES_ONLY; ++j) {
        const int it = vidx(j), s = it % C::NSLOT;
        ok = wait_bar(smem_u32(&bars->kv_full[s]), (it / C::NSLOT) & 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        ok = wait_bar(smem_u32(&bars->p_full[j & 1]), (j >> 1) & 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dv = dV0 + (uint64_t)(s * (C::TILE >> 4));
        const uint32_t acc0 = (j > 0) ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 32 keys per MMA: 32 rows x 128 B of V
          // keys [32 kk, 32 kk + 32): part 32 kk / CW, P8 at its first columns
          const uint32_t col = (32 * kk / C::CW) * C::CW + (32 * kk % C::CW) / 4;
          mma_i8_ts(tbase + 256, tbase + (j & 1) * 128 + col, dv + (uint64_t)(kk * (4096 >> 4)), C::ID_PV,
                    kk > 0 ? 1u : acc0);
        }
        tc_commit(smem_u32(&bars->pv_done));
        tc_commit(smem_u32(&bars->kv_empty[s]));
        if (j == n - 1) tc_commit(smem_u32(&bars->o_full));
        if (j + 2 < n) ok = issue_S(j + 2);
      }
      if (SCORES_ONLY) {
        for (int j = 2; j < n && ok; ++j) {
          // the score buffer of j is free once the softmax warps read block j-2
          ok = wait_bar(smem_u32(&bars->p_full[j & 1]), ((j - 2) >> 1) & 1, abort_flag, p.timeout_ns);
          if (ok) ok = issue_S(j);
        }
      }
      if (!ok) {
        tc_commit(smem_u32(&bars->drain));
        wait_bar_drain(smem_u32(&bars->drain), 0, p.timeout_ns);
      }
    }
    __syncwarp();
  } else {
    // ================================================================ softmax
    constexpr int NCH = C::NCH, CW = C::CW, KPL = CW / 32;  // 32-column chunks, columns, keys per lane
    const int part = (warp - 2) >> 2;  // key columns [CW part, CW part + CW) of every block
    const int quarter = warp & 3;
    const int rr = quarter * 32 + lane;
    const int row = r0 + rr;
    const int cb = part * CW;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tACC = tbase + lane_off + 256 + cb;
    const uint32_t tOF = tbase + lane_off + 384 + cb;
    // exchange slots: [0], [1] row max of even / odd blocks, [2] final l share;
    // each [NPART][128 rows]
    unsigned long long* xch = reinterpret_cast<unsigned long long*>(smem + C::XCH_OFF);
    const int off = p.Nkv - p.Nq;
    const float qs_row = (!SCORES_ONLY && row < p.Nq) ? p.q_scale[(size_t)bh * p.Nq + row] : 0.f;
    const float sv127 = SCORES_ONLY ? 0.f : p.v_scale[bh] * (1.f / 127.f);
    const float* ksrow = p.k_scale + (size_t)bh * p.Nkv;
    // Per-column constants of a key block, kc = s_K * scale * log2(e), kept in
    // this warp's own shared buffer (x / s_Q = S * kc).  Lane l owns columns
    // cb + [KPL l, KPL l + KPL); the next block's scales are loaded one block ahead.
    float* kcbuf = reinterpret_cast<float*>(smem + C::KC_OFF) + (warp - 2) * (2 * CW);
    float ks_next[KPL];
    auto load_ks = [&](int jj) {
      const int c0 = jj * 128 + cb + lane * KPL;
      if (KPL == 2 && p.ks_vec && c0 + 1 < p.Nkv) {
        const float2 v2 = __ldg(reinterpret_cast<const float2*>(ksrow + c0));
        ks_next[0] = v2.x;
        ks_next[KPL - 1] = v2.y;
      } else {
#pragma unroll
        for (int k = 0; k < KPL; ++k) ks_next[k] = (c0 + k < p.Nkv) ? ksrow[c0 + k] : 0.f;
      }
    };
    auto stage_ks = [&](int jj) {
#pragma unroll
      for (int k = 0; k < KPL; ++k) kcbuf[(jj & 1) * CW + lane * KPL + k] = ks_next[k] * p.sl2;
    };
    if (!SCORES_ONLY && n > 0) {
      load_ks(0);
      stage_ks(0);
      if (n > 1) load_ks(1);
      __syncwarp();
    }
    float m_ref = -INFINITY, l = 0.f;  // l: this thread's share (its CW columns)
    bool ok = true;
    if (!SCORES_ONLY) {
      uint32_t z[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] = 0u;
#pragma unroll
      for (int cc = 0; cc < NCH; ++cc) tmem_st32(tOF + cc * 32, z);
      tmem_st_wait();
    }
    for (int j = 0; j < n && ok; ++j) {
      const int kb = j * 128;
      ok = wait_bar(smem_u32(&bars->s_full[j & 1]), (j >> 1) & 1, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tS = tbase + lane_off + (j & 1) * 128 + cb;
      uint32_t s[NCH][32];
#pragma unroll
      for (int c = 0; c < NCH; ++c) tmem_ld32(tS + c * 32, s[c]);
#pragma unroll
      for (int c = 0; c < NCH; ++c) tmem_ld_wait(s[c]);
      if (SCORES_ONLY) {
        if (row < p.Nq) {
          int* dst = p.s_out + ((size_t)bh * p.Nq + row) * p.Nkv + kb + cb;
#pragma unroll
          for (int c = 0; c < NCH; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (kb + cb + c * 32 + i < p.Nkv) dst[c * 32 + i] = (int)s[c][i];
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&bars->p_full[j & 1]));
        continue;
      }
      // y = S * s_K * scale * log2e (= x / s_Q), masked; x = y * s_Q
      const bool tail = kb + 128 > p.Nkv;
      const bool diag = p.causal && (kb + 127 > r0 + off);
      int lim = 127;
      if (tail || diag) {
        lim = p.Nkv - 1 - kb;
        if (p.causal) lim = min(lim, row + off - kb);
      }
      lim -= cb;
      const float* kcb = kcbuf + (j & 1) * CW;
      float x[NCH][32];
      const uint64_t negM2 = f2(-12582912.f, -12582912.f);
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 kc = *reinterpret_cast<const float4*>(kcb + c * 32 + i);
          // exact int32 -> fp32 (|S| < 2^22): bits of 1.5 * 2^23 + S, minus 1.5 * 2^23
          const uint64_t sa = fadd2(f2(__int_as_float((int)s[c][i + 0] + 0x4B400000),
                                       __int_as_float((int)s[c][i + 1] + 0x4B400000)), negM2);
          const uint64_t sb = fadd2(f2(__int_as_float((int)s[c][i + 2] + 0x4B400000),
                                       __int_as_float((int)s[c][i + 3] + 0x4B400000)), negM2);
          f2_split(fmul2(sa, f2(kc.x, kc.y)), x[c][i + 0], x[c][i + 1]);
          f2_split(fmul2(sb, f2(kc.z, kc.w)), x[c][i + 2], x[c][i + 3]);
        }
      }
      if (tail || diag) {
#pragma unroll
        for (int c = 0; c < NCH; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i > lim) x[c][i] = -INFINITY;
      }
      // the next block's scales go to the other buffer while this one is in use
      if (j + 1 < n) {
        stage_ks(j + 1);
        if (j + 2 < n) load_ks(j + 2);
      }
      float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
      for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          mxa = fmax3(mxa, x[c][i], x[c][i + 1]);
          mxb = fmax3(mxb, x[c][i + 2], x[c][i + 3]);
        }
      // row max over the NPART parts.  Slot j % 2 is rewritten for block j + 2
      // only after this thread read every partner's block j + 1 value, which
      // each partner writes after reading ours for block j.
      const float my_max = fmaxf(mxa, mxb);
      float row_max = my_max;
      unsigned long long* xj = xch + (j & 1) * (C::NPART * 128);
      xchg_put(xj + part * 128 + rr, (uint32_t)j + 1u, my_max);
#pragma unroll
      for (int q = 1; q < C::NPART; ++q) {
        float other;
        const int pq = (part + q) % C::NPART;
        ok = ok && xchg_get(xj + pq * 128 + rr, (uint32_t)j + 1u, other, abort_flag, p.timeout_ns);
        row_max = fmaxf(row_max, ok ? other : row_max);
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      // s_Q > 0, so max(y) * s_Q is the row max of x
      const float m_blk = row_max * qs_row;
      // tau = 0: move the reference on every increase
      const bool grow = m_blk > m_ref;
      const bool had = m_ref != -INFINITY;  // rows with earlier content need a fold
      float factor = 1.f;
      if (grow) {
        factor = had ? ex2(m_ref - m_blk) : 0.f;
        l *= factor;
        m_ref = m_blk;
      }
      // P8 = rne(127 * 2^(x - m)) = rne(2^(x - m + log2 127)); the rounding is
      // the low byte of 1.5 * 2^23 + y
      const float negm = ((m_ref == -INFINITY) ? 0.f : -m_ref) + 6.9886846867721655f;
      const uint64_t qs2 = f2(qs_row, qs_row), nm2 = f2(negm, negm);
      const uint64_t mg2 = f2(12582912.f, 12582912.f);
      uint32_t isum = 0;
      uint32_t pk[CW / 4];
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          float a0, a1, a2, a3;
          f2_split(ffma2(f2(x[c][i + 0], x[c][i + 1]), qs2, nm2), a0, a1);
          f2_split(ffma2(f2(x[c][i + 2], x[c][i + 3]), qs2, nm2), a2, a3);
          float t0, t1, t2, t3;
          f2_split(fadd2(f2(ex2(a0), ex2(a1)), mg2), t0, t1);
          f2_split(fadd2(f2(ex2(a2), ex2(a3)), mg2), t2, t3);
          const uint32_t lo = __byte_perm(__float_as_uint(t0), __float_as_uint(t1), 0x0040);
          const uint32_t hi = __byte_perm(__float_as_uint(t2), __float_as_uint(t3), 0x0040);
          const uint32_t w = __byte_perm(lo, hi, 0x5410);
          pk[c * 8 + i / 4] = w;
          isum = __dp4a(w, 0x01010101u, isum);
        }
      }
      l += (float)isum * (1.f / 127.f);
      // P8 of keys [cb, cb + CW) -> columns [cb, cb + CW / 4) of this block's score buffer
      if (CW == 32) {
        tmem_st8(tS, pk);
      } else {
        uint32_t p16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) p16[i] = pk[i % (CW / 4)];
        tmem_st16(tS, p16);
      }
      if (j > 0 && __any_sync(0xffffffffu, grow && had)) {
        // fold ACC (P V of blocks < j, reference m_old) into OF
        ok = wait_bar(smem_u32(&bars->pv_done), (j - 1) & 1, abort_flag, p.timeout_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const float f = (grow && had) ? factor : 1.f;
        // every chunk of ACC and OF requested before the first wait (one
        // tensor-memory round trip instead of one per chunk)
        uint32_t a[NCH][32], o[NCH][32];
#pragma unroll
        for (int cc = 0; cc < NCH; ++cc) {
          tmem_ld32(tACC + cc * 32, a[cc]);
          tmem_ld32(tOF + cc * 32, o[cc]);
        }
#pragma unroll
        for (int cc = 0; cc < NCH; ++cc) {
          tmem_ld_wait(a[cc]);
          tmem_ld_wait(o[cc]);
        }
#pragma unroll
        for (int cc = 0; cc < NCH; ++cc) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            o[cc][i] = __float_as_uint((__uint_as_float(o[cc][i]) + (float)(int)a[cc][i] * sv127) * f);
            a[cc][i] = 0u;
          }
          tmem_st32(tOF + cc * 32, o[cc]);
          tmem_st32(tACC + cc * 32, a[cc]);
        }
      }
      tmem_st_wait();
      __syncwarp();  // the staged scales of block j + 1 are visible to the whole warp
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->p_full[j & 1]));
    }
    // ---------------------------------------------------------- epilogue
    if (!SCORES_ONLY && ok) {
      ok = wait_bar(smem_u32(&bars->o_full), 0, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (!SCORES_ONLY && ok) {
      unsigned long long* xl = xch + 2 * (C::NPART * 128);
      xchg_put(xl + part * 128 + rr, 1u, l);
      float lt = l;
#pragma unroll
      for (int q = 1; q < C::NPART; ++q) {
        float other;
        const int pq = (part + q) % C::NPART;
        ok = ok && xchg_get(xl + pq * 128 + rr, 1u, other, abort_flag, p.timeout_ns);
        lt += ok ? other : 0.f;
      }
      ok = __all_sync(0xffffffffu, ok);
      l = lt;
    }
    if (!SCORES_ONLY && ok) {
      tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      float* orow = p.o + ((size_t)bh * p.Nq + row) * C::D + cb;
#pragma unroll 1
      for (int cc = 0; cc < NCH; ++cc) {
        uint32_t a[32], o[32];
        tmem_ld32(tACC + cc * 32, a);
        tmem_ld32(tOF + cc * 32, o);
        tmem_ld_wait(a);
        tmem_ld_wait(o);
        if (row < p.Nq) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            float4 v;
            v.x = (l > 0.f) ? (__uint_as_float(o[i + 0]) + (float)(int)a[i + 0] * sv127) * inv : 0.f;
            v.y = (l > 0.f) ? (__uint_as_float(o[i + 1]) + (float)(int)a[i + 1] * sv127) * inv : 0.f;
            v.z = (l > 0.f) ? (__uint_as_float(o[i + 2]) + (float)(int)a[i + 2] * sv127) * inv : 0.f;
            v.w = (l > 0.f) ? (__uint_as_float(o[i + 3]) + (float)(int)a[i + 3] * sv127) * inv : 0.f;
            *reinterpret_cast<float4*>(orow + cc * 32 + i) = v;
          }
        }
      }
      if (part == 0 && row < p.Nq)
        p.lse[(size_t)bh * p.Nq + row] = (l > 0.f) ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace ta
