// bf16 attention backward for sm_100a (TMA + tcgen05 + TMEM), by recomputation.
//
// "Can a full-day context beat one minute? Flash attention and the
// sequence-length question", section "Backward: recompute instead of store":
// the backward needs P, which the forward never stores; it is recomputed tile
// by tile from Q, K and the softmax statistics kept by the forward (here the
// LSE), and only O (for the row statistic below) is read besides the inputs.
// With S = scale Q K^T (masked) and P = exp(S - LSE):
//   dV = P^T dO,  dP = dO V^T,  dS = P o (dP - Dr),  Dr_i = sum_c dO_ic O_ic,
//   dQ = scale dS K,  dK = scale dS^T Q.
// Three kernels:
//   bwd_rowdot_kernel  Dr per query row (one warp per row);
//   bwd_dkdv_kernel    one CTA per (batch*head, 128-key tile): walks the
//                      query tiles, computes S^T = K Q^T and dP^T = V dO^T in
//                      TMEM (thread = key row), turns them into P^T and dS^T
//                      (bf16, written back into the same TMEM columns), and
//                      accumulates dV += P^T dO and dK += dS^T Q with P^T and
//                      dS^T as TMEM A operands;
//   bwd_dq_kernel      one CTA per (batch*head, 128-query tile): walks the key
//                      tiles, S = Q K^T and dP = dO V^T, dS in TMEM, and
//                      dQ += dS K.
// FP8-P variant (P8 = true; "Hardware-Aware FP4 FlashAttention-4" page: in
// training, 4-bit probabilities made the backward diverge and 8-bit ones kept
// it stable): the recomputed P is rounded to e4m3 (unit scale, P <= 1) before
// it enters dV = P^T dO; dS uses P unrounded.  e4m3 values are exact in bf16,
// so the bf16 MMA computes exactly the product with the 8-bit P.
// Each kernel: warp 0 TMA producer, warp 1 MMA issuer (one thread), warps 2-5
// compute (thread = TMEM lane).  The score pair of a tile is computed, turned
// into P / dS, then the accumulating MMAs run; the next tile's scores are
// issued after them (their TMEM columns are reused).
#pragma once
#include "ptx.cuh"
#include "fwd_bf16.cuh"  // FwdCfg tile geometry, fwd_tile_kv_count, wait_bar_drain

namespace ta {

struct BwdParams {
  const uint16_t* o;     // [BH][Nq][D] forward output
  const uint16_t* dout;  // [BH][Nq][D] upstream gradient
  const float* lse;      // [BH][Nq] natural-log LSE from the forward
  float* rowdot;         // [BH][Nq] Dr = sum_c dO O (workspace)
  uint16_t* dq;          // [BH][Nq][D]
  uint16_t* dk;          // [BH][Nkv][D]
  uint16_t* dv;          // [BH][Nkv][D]
  int Nq, Nkv, nqt, nkt;  // tiles of 128 queries / keys
  int causal;
  float scale, sl2;  // scale, scale * log2(e)
  unsigned long long timeout_ns;
};

// Dr_i = sum_c dO_ic O_ic (fp32), one warp per row.
template <int D>
__global__ void __launch_bounds__(256) bwd_rowdot_kernel(const uint16_t* __restrict__ o,
                                                         const uint16_t* __restrict__ dout,
                                                         float* __restrict__ rowdot, long long rows) {
  constexpr int E = D / 32;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    const uint32_t a = *reinterpret_cast<const uint32_t*>(o + row * D + lane * E + e);
    const uint32_t b = *reinterpret_cast<const uint32_t*>(dout + row * D + lane * E + e);
    acc = fmaf(__uint_as_float(a << 16), __uint_as_float(b << 16), acc);
    acc = fmaf(__uint_as_float(a & 0xFFFF0000u), __uint_as_float(b & 0xFFFF0000u), acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) rowdot[row] = acc;
}

template <int D>
struct BwdCfg {
  static constexpr int TILE = 128 * D * 2;  // one 128 x D bf16 tile
  static constexpr int HALF = 128 * 128;    // one 64-column block of a tile
  static constexpr int NST = 2;             // ring stages (two tiles each)
  static constexpr int STAGE = 2 * TILE;
  static constexpr int FIX_OFF = 0;                   // the tile pair kept for the whole CTA
  static constexpr int ST_OFF = 2 * TILE;             // ring of tile pairs
  static constexpr int COL_OFF = ST_OFF + NST * STAGE;  // dkdv: per-warp LSE / Dr columns [4][2][128]
  static constexpr int BAR_OFF = COL_OFF + 4 * 2 * 128 * 4;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
  static constexpr int THREADS = 192;
  static constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, false);  // 128 x 128 scores
  static constexpr uint32_t ID_ACC = idesc_bf16_f32(128, D, true);   // accumulate, B MN-major
};

struct BwdBars {
  uint64_t fix_full;
  uint64_t st_full[2];
  uint64_t st_empty[2];
  uint64_t s_full;   // scores of the current tile pair in TMEM
  uint64_t p_full;   // P / dS written back (count 128)
  uint64_t acc_full; // accumulators final
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(BwdBars) <= 256, "barrier block too large");

// Score MMAs of one tile pair: D0 = A0 B0^T, D1 = A1 B1^T (K-major operands).
template <int D>
__device__ __forceinline__ void bwd_issue_scores(uint32_t d0, uint32_t d1, uint64_t a0, uint64_t b0, uint64_t a1,
                                                 uint64_t b1) {
  using C = BwdCfg<D>;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = (uint64_t)(((kk >> 2) * C::HALF + (kk & 3) * 32) >> 4);
    mma_f16_ss(d0, a0 + off, b0 + off, C::ID_S, kk > 0);
  }
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = (uint64_t)(((kk >> 2) * C::HALF + (kk & 3) * 32) >> 4);
    mma_f16_ss(d1, a1 + off, b1 + off, C::ID_S, kk > 0);
  }
}
// Accumulating MMA: Dacc (+)= A(tmem, 128 x 128 bf16) B(smem tile, MN-major).
template <int D>
__device__ __forceinline__ void bwd_issue_acc(uint32_t dacc, uint32_t a_tmem, uint64_t b, bool accumulate) {
  using C = BwdCfg<D>;
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk)
    mma_f16_ts(dacc, a_tmem + kk * 8, b + (uint64_t)(kk * (2048 >> 4)), C::ID_ACC, (accumulate || kk > 0) ? 1u : 0u);
}

// Rows of a [128 x D] fp32 accumulator in TMEM (this thread's lane) -> bf16
// global row, times `mul`.
template <int D>
__device__ __forceinline__ void bwd_store_row(uint32_t tacc, uint16_t* dst, float mul, bool write) {
#pragma unroll 1
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t a[32];
    tmem_ld32(tacc + cc * 32, a);
    tmem_ld_wait(a);
    if (write) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          w[e] = pack_bf16(__uint_as_float(a[g * 8 + 2 * e]) * mul, __uint_as_float(a[g * 8 + 2 * e + 1]) * mul);
        *reinterpret_cast<uint4*>(dst + cc * 32 + g * 8) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

// a pair of non-negative floats rounded to e4m3 (RNE, saturating), as bf16x2
__device__ __forceinline__ uint32_t e4m3_round_bf16x2(float lo, float hi) {
  uint32_t h2;
  asm("{\n\t.reg .b16 c;\n\tcvt.rn.satfinite.e4m3x2.f32 c, %1, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}"
      : "=r"(h2)
      : "f"(hi), "f"(lo));
  float a, b;
  asm("{\n\t.reg .b16 x, y;\n\tmov.b32 {x, y}, %2;\n\tcvt.f32.f16 %0, x;\n\tcvt.f32.f16 %1, y;\n\t}"
      : "=f"(a), "=f"(b)
      : "r"(h2));
  return pack_bf16(a, b);  // exact: every e4m3 value is a bf16 value
}

// P = exp2(S * sl2 - lse2) and dS = P (dP - Dr) for 32 columns, packed bf16x2
// (P8: the P words hold e4m3-rounded P).
template <bool P8 = false>
__device__ __forceinline__ void bwd_p_ds(const uint32_t (&s)[32], const uint32_t (&dp)[32], const float* lse2,
                                         const float* rd, float sl2, uint32_t vis_mask, uint32_t (&pp)[16],
                                         uint32_t (&pd)[16]) {
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    float p0 = ex2(fmaf(__uint_as_float(s[i]), sl2, -lse2[i]));
    float p1 = ex2(fmaf(__uint_as_float(s[i + 1]), sl2, -lse2[i + 1]));
    p0 = ((vis_mask >> i) & 1u) ? p0 : 0.f;
    p1 = ((vis_mask >> (i + 1)) & 1u) ? p1 : 0.f;
    const float d0 = p0 * (__uint_as_float(dp[i]) - rd[i]);
    const float d1 = p1 * (__uint_as_float(dp[i + 1]) - rd[i + 1]);
    if constexpr (P8)
      pp[i / 2] = e4m3_round_bf16x2(p0, p1);
    else
      pp[i / 2] = pack_bf16(p0, p1);
    pd[i / 2] = pack_bf16(d0, d1);
  }
}

// visible columns [c0, c0 + 32) of a row: key k sees query q iff q < Nq,
// k < Nkv and (not causal or k <= q + Nkv - Nq)
__device__ __forceinline__ uint32_t bwd_mask32(int lo, int hi) {  // bits [lo, hi) within 0..31
  lo = max(lo, 0);
  hi = min(hi, 32);
  if (hi <= lo) return 0u;
  const uint32_t upto = (hi >= 32) ? 0xFFFFFFFFu : ((1u << hi) - 1u);
  return upto & ~((1u << lo) - 1u);
}

// ============================================================== dK, dV
template <int D, bool P8 = false>
__global__ void __launch_bounds__(192, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::BAR_OFF);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = (int)blockIdx.x / p.nkt, kt = (int)blockIdx.x % p.nkt;
  const int k0 = kt * 128;
  const int off = p.Nkv - p.Nq;
  // query tiles that see some key of this tile: q >= k0 - off
  const int first_q = p.causal ? max(0, k0 - off) : 0;
  const int it0 = first_q / 128;
  const int nit = (first_q < p.Nq) ? p.nqt - it0 : 0;
  volatile int* abort_flag = &bars->abort;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->fix_full), 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(smem_u32(&bars->st_full[s]), 1);
      mbar_init(smem_u32(&bars->st_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->s_full), 1);
    mbar_init(smem_u32(&bars->p_full), 128);
    mbar_init(smem_u32(&bars->acc_full), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;
  // TMEM: S^T [0,128) (P^T bf16 in [0,64)), dP^T [128,256) (dS^T in [128,192)),
  // dV [256, 256+D), dK [256+D, 256+2D)
  const uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + D;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmDO);
      const uint32_t fb = smem_u32(&bars->fix_full);
      mbar_arrive_expect_tx(fb, 2 * C::TILE);
      for (int h = 0; h < D / 64; ++h) {
        tma_load_3d(sbase + C::FIX_OFF + h * C::HALF, &tmK, fb, h * 64, k0, bh);
        tma_load_3d(sbase + C::FIX_OFF + C::TILE + h * C::HALF, &tmV, fb, h * 64, k0, bh);
      }
      bool ok = true;
      int t = 0;
      for (; t < nit && ok; ++t) {
        const int s = t % C::NST;
        const uint32_t ph = (t / C::NST) & 1;
        ok = wait_bar(smem_u32(&bars->st_empty[s]), ph ^ 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        const uint32_t sb = smem_u32(&bars->st_full[s]);
        mbar_arrive_expect_tx(sb, 2 * C::TILE);
        const uint32_t dst = sbase + C::ST_OFF + s * C::STAGE;
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(dst + h * C::HALF, &tmQ, sb, h * 64, (it0 + t) * 128, bh);
          tma_load_3d(dst + C::TILE + h * C::HALF, &tmDO, sb, h * 64, (it0 + t) * 128, bh);
        }
      }
      if (!ok) {
        wait_bar_drain(fb, 0, p.timeout_ns);
        for (int back = 1; back <= C::NST && t - back >= 0; ++back) {
          const int i2 = t - back;
          wait_bar_drain(smem_u32(&bars->st_full[i2 % C::NST]), (i2 / C::NST) & 1, p.timeout_ns);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = wait_bar(smem_u32(&bars->fix_full), 0, abort_flag, p.timeout_ns);
      tc_fence_after();
      const uint64_t dK = smem_desc(sbase + C::FIX_OFF, 16, 1024);
      const uint64_t dV = smem_desc(sbase + C::FIX_OFF + C::TILE, 16, 1024);
      for (int t = 0; t < nit && ok; ++t) {
        const int s = t % C::NST;
        ok = wait_bar(smem_u32(&bars->st_full[s]), (t / C::NST) & 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        const uint32_t st = sbase + C::ST_OFF + s * C::STAGE;
        // S^T = K Q_i^T, dP^T = V dO_i^T
        bwd_issue_scores<D>(tbase + T_S, tbase + T_DP, dK, smem_desc(st, 16, 1024), dV,
                            smem_desc(st + C::TILE, 16, 1024));
        tc_commit(smem_u32(&bars->s_full));
        ok = wait_bar(smem_u32(&bars->p_full), t & 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        // dV += P^T dO_i, dK += dS^T Q_i (B operands MN-major: keys of the
        // contraction are the tile's rows)
        bwd_issue_acc<D>(tbase + T_DV, tbase + T_S, smem_desc(st + C::TILE, C::HALF, 1024), t > 0);
        bwd_issue_acc<D>(tbase + T_DK, tbase + T_DP, smem_desc(st, C::HALF, 1024), t > 0);
        tc_commit(smem_u32(&bars->st_empty[s]));
      }
      if (ok) tc_commit(smem_u32(&bars->acc_full));
      if (!ok) {
        tc_commit(smem_u32(&bars->drain));
        wait_bar_drain(smem_u32(&bars->drain), 0, p.timeout_ns);
      }
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3;
    const int rr = quarter * 32 + lane;
    const int key = k0 + rr;  // this thread's key row
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    float* cols = reinterpret_cast<float*>(smem + C::COL_OFF) + (warp - 2) * 256;  // [lse2 128][rd 128]
    const float* lse_bh = p.lse + (size_t)bh * p.Nq;
    const float* rd_bh = p.rowdot + (size_t)bh * p.Nq;
    bool ok = true;
    for (int t = 0; t < nit && ok; ++t) {
      const int q0 = (it0 + t) * 128;
      // column statistics of this query tile, per warp: LSE in log2 units
      // (+inf past the end, so that P = 0) and Dr
      __syncwarp();
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int q = q0 + lane * 4 + e;
        cols[lane * 4 + e] = (q < p.Nq) ? lse_bh[q] * 1.4426950408889634f : INFINITY;
        cols[128 + lane * 4 + e] = (q < p.Nq) ? rd_bh[q] : 0.f;
      }
      __syncwarp();
      ok = wait_bar(smem_u32(&bars->s_full), t & 1, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t s[32], dp[32];
        tmem_ld32(tbase + lane_off + T_S + c * 32, s);
        tmem_ld32(tbase + lane_off + T_DP + c * 32, dp);
        tmem_ld_wait(s);
        tmem_ld_wait(dp);
        // visible: q < Nq, key < Nkv, and (causal) q >= key - off
        int lo = 0, hi = p.Nq - (q0 + c * 32);
        if (key >= p.Nkv) hi = 0;
        if (p.causal) lo = key - off - (q0 + c * 32);
        const uint32_t vis = bwd_mask32(lo, hi);
        uint32_t pp[16], pd[16];
        bwd_p_ds<P8>(s, dp, cols + c * 32, cols + 128 + c * 32, p.sl2, vis, pp, pd);
        // P^T and dS^T over columns already read (16 words land in the first
        // half of the 32 columns this chunk index has passed)
        tmem_st16(tbase + lane_off + T_S + c * 16, pp);
        tmem_st16(tbase + lane_off + T_DP + c * 16, pd);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->p_full));
    }
    if (ok) {
      ok = wait_bar(smem_u32(&bars->acc_full), 0, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const bool w = key < p.Nkv;
      if (nit > 0) {
        bwd_store_row<D>(tbase + lane_off + T_DV, p.dv + ((size_t)bh * p.Nkv + key) * D, 1.f, w);
        bwd_store_row<D>(tbase + lane_off + T_DK, p.dk + ((size_t)bh * p.Nkv + key) * D, p.scale, w);
      } else if (w) {  // no query sees these keys
        for (int e = 0; e < D; e += 8) {
          *reinterpret_cast<uint4*>(p.dv + ((size_t)bh * p.Nkv + key) * D + e) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(p.dk + ((size_t)bh * p.Nkv + key) * D + e) = make_uint4(0, 0, 0, 0);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ============================================================== dQ
template <int D>
__global__ void __launch_bounds__(192, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::BAR_OFF);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = (int)blockIdx.x / p.nqt, qt = (int)blockIdx.x % p.nqt;
  const int q0 = qt * 128;
  const int nj = fwd_tile_kv_count(q0, p.Nq, p.Nkv, p.nkt, p.causal);
  const int off = p.Nkv - p.Nq;
  volatile int* abort_flag = &bars->abort;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->fix_full), 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(smem_u32(&bars->st_full[s]), 1);
      mbar_init(smem_u32(&bars->st_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->s_full), 1);
    mbar_init(smem_u32(&bars->p_full), 128);
    mbar_init(smem_u32(&bars->acc_full), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;
  // TMEM: S [0,128), dP [128,256) (dS bf16 in [128,192)), dQ [256, 256+D)
  const uint32_t T_S = 0, T_DP = 128, T_DQ = 256;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmDO);
      const uint32_t fb = smem_u32(&bars->fix_full);
      mbar_arrive_expect_tx(fb, 2 * C::TILE);
      for (int h = 0; h < D / 64; ++h) {
        tma_load_3d(sbase + C::FIX_OFF + h * C::HALF, &tmQ, fb, h * 64, q0, bh);
        tma_load_3d(sbase + C::FIX_OFF + C::TILE + h * C::HALF, &tmDO, fb, h * 64, q0, bh);
      }
      bool ok = true;
      int t = 0;
      for (; t < nj && ok; ++t) {
        const int s = t % C::NST;
        const uint32_t ph = (t / C::NST) & 1;
        ok = wait_bar(smem_u32(&bars->st_empty[s]), ph ^ 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        const uint32_t sb = smem_u32(&bars->st_full[s]);
        mbar_arrive_expect_tx(sb, 2 * C::TILE);
        const uint32_t dst = sbase + C::ST_OFF + s * C::STAGE;
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(dst + h * C::HALF, &tmK, sb, h * 64, t * 128, bh);
          tma_load_3d(dst + C::TILE + h * C::HALF, &tmV, sb, h * 64, t * 128, bh);
        }
      }
      if (!ok) {
        wait_bar_drain(fb, 0, p.timeout_ns);
        for (int back = 1; back <= C::NST && t - back >= 0; ++back) {
          const int i2 = t - back;
          wait_bar_drain(smem_u32(&bars->st_full[i2 % C::NST]), (i2 / C::NST) & 1, p.timeout_ns);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = wait_bar(smem_u32(&bars->fix_full), 0, abort_flag, p.timeout_ns);
      tc_fence_after();
      const uint64_t dQ = smem_desc(sbase + C::FIX_OFF, 16, 1024);
      const uint64_t dDO = smem_desc(sbase + C::FIX_OFF + C::TILE, 16, 1024);
      for (int t = 0; t < nj && ok; ++t) {
        const int s = t % C::NST;
        ok = wait_bar(smem_u32(&bars->st_full[s]), (t / C::NST) & 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        const uint32_t st = sbase + C::ST_OFF + s * C::STAGE;
        // S = Q K_j^T, dP = dO V_j^T
        bwd_issue_scores<D>(tbase + T_S, tbase + T_DP, dQ, smem_desc(st, 16, 1024), dDO,
                            smem_desc(st + C::TILE, 16, 1024));
        tc_commit(smem_u32(&bars->s_full));
        ok = wait_bar(smem_u32(&bars->p_full), t & 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        // dQ += dS K_j (K_j rows are the contraction: B MN-major)
        bwd_issue_acc<D>(tbase + T_DQ, tbase + T_DP, smem_desc(st, C::HALF, 1024), t > 0);
        tc_commit(smem_u32(&bars->st_empty[s]));
      }
      if (ok) tc_commit(smem_u32(&bars->acc_full));
      if (!ok) {
        tc_commit(smem_u32(&bars->drain));
        wait_bar_drain(smem_u32(&bars->drain), 0, p.timeout_ns);
      }
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3;
    const int rr = quarter * 32 + lane;
    const int row = q0 + rr;  // this thread's query row
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const bool live = row < p.Nq;
    const float lse2 = live ? p.lse[(size_t)bh * p.Nq + row] * 1.4426950408889634f : INFINITY;
    const float rd = live ? p.rowdot[(size_t)bh * p.Nq + row] : 0.f;
    float lse2v[32], rdv[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      lse2v[i] = lse2;
      rdv[i] = rd;
    }
    bool ok = true;
    for (int t = 0; t < nj && ok; ++t) {
      const int kb = t * 128;
      ok = wait_bar(smem_u32(&bars->s_full), t & 1, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t s[32], dp[32];
        tmem_ld32(tbase + lane_off + T_S + c * 32, s);
        tmem_ld32(tbase + lane_off + T_DP + c * 32, dp);
        tmem_ld_wait(s);
        tmem_ld_wait(dp);
        // visible keys: k < Nkv and (causal) k <= row + off
        int hi = p.Nkv - (kb + c * 32);
        if (p.causal) hi = min(hi, row + off - (kb + c * 32) + 1);
        if (!live) hi = 0;
        const uint32_t vis = bwd_mask32(0, hi);
        uint32_t pp[16], pd[16];
        bwd_p_ds(s, dp, lse2v, rdv, p.sl2, vis, pp, pd);
        tmem_st16(tbase + lane_off + T_DP + c * 16, pd);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->p_full));
    }
    if (ok) {
      ok = wait_bar(smem_u32(&bars->acc_full), 0, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      uint16_t* dst = p.dq + ((size_t)bh * p.Nq + row) * D;
      if (nj > 0) {
        bwd_store_row<D>(tbase + lane_off + T_DQ, dst, p.scale, live);
      } else if (live) {  // no key visible to this tile
        for (int e = 0; e < D; e += 8) *reinterpret_cast<uint4*>(dst + e) = make_uint4(0, 0, 0, 0);
      }
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
