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
// Each kernel: warp 0 TMA producer, warp 1 MMA issuer (one thread), warps
// 2-17 compute: four warps per TMEM lane quarter (thread = lane = row of the
// tile), each over 32 of the 128 columns, since P and dS are elementwise and
// need no row reduction.  The two score groups of a tile have their own
// barriers and the compute warps work in two phases, P from S first (kept in
// fp32 registers), then dS from dP, so that the tensor core never waits for a
// whole tile: dkdv issues S^T(t), dP^T(t) | dV(t), S^T(t+1) | dK(t), dP^T(t+1)
// and dq issues S(t), dP(t) | S(t+1) | dQ(t), dP(t+1), each group as soon as
// the compute phase it depends on has released its TMEM columns.
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
  // compute warps: 4 per TMEM lane quarter, one 32-column chunk of the tile each
  static constexpr int NCW = 16;
  static constexpr int COL_OFF = ST_OFF + NST * STAGE;  // dkdv: per-warp LSE / Dr of its chunk [16][2][32]
  static constexpr int BAR_OFF = COL_OFF + NCW * 2 * 32 * 4;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
  static constexpr int THREADS = 64 + NCW * 32;  // producer, MMA issuer, compute warps
  static constexpr int CT = NCW * 32;            // compute threads (barrier counts)
  static constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, false);  // 128 x 128 scores
  static constexpr uint32_t ID_ACC = idesc_bf16_f32(128, D, true);   // accumulate, B MN-major
};

struct BwdBars {
  uint64_t fix_full;
  uint64_t st_full[2];
  uint64_t st_empty[2];
  uint64_t s_full;   // S (S^T) of the current tile in TMEM
  uint64_t dp_full;  // dP (dP^T) of the current tile in TMEM
  uint64_t p_full;   // dkdv: P^T written back; dq: S read (all compute threads)
  uint64_t ds_full;  // dS (dS^T) written back (all compute threads)
  uint64_t s_read;   // dkdv: every compute thread holds its S^T chunk (P^T words may land)
  uint64_t dp_read;  // dkdv: every compute thread holds its dP^T chunk
  uint64_t acc_full; // accumulators final
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(BwdBars) <= 256, "barrier block too large");

// One score MMA group: D = A B^T (128 x 128, K-major operands).
template <int D>
__device__ __forceinline__ void bwd_issue_score(uint32_t d, uint64_t a, uint64_t b) {
  using C = BwdCfg<D>;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = (uint64_t)(((kk >> 2) * C::HALF + (kk & 3) * 32) >> 4);
    mma_f16_ss(d, a + off, b + off, C::ID_S, kk > 0);
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

// 32 columns of a [128 x D] fp32 accumulator in TMEM (this thread's lane) ->
// 32 bf16 of a global row, times `mul` (write = false: TMEM read only; the
// load is warp-collective).
__device__ __forceinline__ void bwd_store_chunk(uint32_t tacc, uint16_t* dst, float mul, bool write) {
  uint32_t a[32];
  tmem_ld32(tacc, a);
  tmem_ld_wait(a);
  if (write) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        w[e] = pack_bf16(__uint_as_float(a[g * 8 + 2 * e]) * mul, __uint_as_float(a[g * 8 + 2 * e + 1]) * mul);
      *reinterpret_cast<uint4*>(dst + g * 8) = make_uint4(w[0], w[1], w[2], w[3]);
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
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
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
    mbar_init(smem_u32(&bars->dp_full), 1);
    mbar_init(smem_u32(&bars->p_full), C::CT);
    mbar_init(smem_u32(&bars->ds_full), C::CT);
    mbar_init(smem_u32(&bars->s_read), C::CT);
    mbar_init(smem_u32(&bars->dp_read), C::CT);
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
      auto stage = [&](int t) { return sbase + C::ST_OFF + (t % C::NST) * C::STAGE; };
      auto stage_full = [&](int t) -> bool {
        const bool r = wait_bar(smem_u32(&bars->st_full[t % C::NST]), (t / C::NST) & 1, abort_flag, p.timeout_ns);
        tc_fence_after();
        return r;
      };
      // S^T(0) = K Q_0^T, dP^T(0) = V dO_0^T
      if (ok && nit > 0 && (ok = stage_full(0))) {
        bwd_issue_score<D>(tbase + T_S, dK, smem_desc(stage(0), 16, 1024));
        tc_commit(smem_u32(&bars->s_full));
        bwd_issue_score<D>(tbase + T_DP, dV, smem_desc(stage(0) + C::TILE, 16, 1024));
        tc_commit(smem_u32(&bars->dp_full));
      }
      for (int t = 0; t < nit && ok; ++t) {
        const uint32_t st = stage(t);
        ok = wait_bar(smem_u32(&bars->p_full), t & 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        // dV += P^T dO_t (B operand MN-major: keys of the contraction are the tile's rows)
        bwd_issue_acc<D>(tbase + T_DV, tbase + T_S, smem_desc(st + C::TILE, C::HALF, 1024), t > 0);
        if (t + 1 < nit) {  // S^T(t+1) over the P^T(t) columns, after the dV MMAs in the pipe
          if (!(ok = stage_full(t + 1))) break;
          bwd_issue_score<D>(tbase + T_S, dK, smem_desc(stage(t + 1), 16, 1024));
          tc_commit(smem_u32(&bars->s_full));
        }
        ok = wait_bar(smem_u32(&bars->ds_full), t & 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        // dK += dS^T Q_t
        bwd_issue_acc<D>(tbase + T_DK, tbase + T_DP, smem_desc(st, C::HALF, 1024), t > 0);
        tc_commit(smem_u32(&bars->st_empty[t % C::NST]));
        if (t + 1 < nit) {  // dP^T(t+1) over the dS^T(t) columns, after the dK MMAs
          bwd_issue_score<D>(tbase + T_DP, dV, smem_desc(stage(t + 1) + C::TILE, 16, 1024));
          tc_commit(smem_u32(&bars->dp_full));
        }
      }
      if (ok) tc_commit(smem_u32(&bars->acc_full));
      if (!ok) {
        tc_commit(smem_u32(&bars->drain));
        wait_bar_drain(smem_u32(&bars->drain), 0, p.timeout_ns);
      }
    }
    __syncwarp();
  } else {
    // compute warp: TMEM lane quarter warp % 4 (its key rows), query columns [32c, 32c + 32)
    const int cw = warp - 2;
    const int quarter = warp & 3, c = cw >> 2;
    const int rr = quarter * 32 + lane;
    const int key = k0 + rr;  // this thread's key row
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    float* cols = reinterpret_cast<float*>(smem + C::COL_OFF) + cw * 64;  // [lse2 32][rd 32] of the chunk
    const float* lse_bh = p.lse + (size_t)bh * p.Nq;
    const float* rd_bh = p.rowdot + (size_t)bh * p.Nq;
    bool ok = true;
    // column statistics of a chunk: LSE in log2 units (+inf past the end, so
    // that P = 0) and Dr; lane i loads column i, one tile ahead of their use
    auto load_stats = [&](int tt, float& ls, float& r) {
      const int q = (it0 + tt) * 128 + 32 * c + lane;
      ls = (q < p.Nq) ? lse_bh[q] * 1.4426950408889634f : INFINITY;
      r = (q < p.Nq) ? rd_bh[q] : 0.f;
    };
    float nls = 0.f, nrd = 0.f;
    if (nit > 0) load_stats(0, nls, nrd);
    for (int t = 0; t < nit && ok; ++t) {
      const int qc = (it0 + t) * 128 + 32 * c;  // first query column of this chunk
      __syncwarp();
      cols[lane] = nls;
      cols[32 + lane] = nrd;
      __syncwarp();
      if (t + 1 < nit) load_stats(t + 1, nls, nrd);
      ok = wait_bar(smem_u32(&bars->s_full), t & 1, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // phase 1: P^T = exp2(S^T sl2 - lse2) (masked), kept in fp32 for dS^T
      float pf[32];
      uint32_t pp[16];
      {
        uint32_t sv[32];
        tmem_ld32(tbase + lane_off + T_S + c * 32, sv);
        tmem_ld_wait(sv);
        // visible: q < Nq, key < Nkv, and (causal) q >= key - off
        int lo = 0, hi = p.Nq - qc;
        if (key >= p.Nkv) hi = 0;
        if (p.causal) lo = key - off - qc;
        const uint32_t vis = bwd_mask32(lo, hi);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float p0 = ((vis >> i) & 1u) ? ex2(fmaf(__uint_as_float(sv[i]), p.sl2, -cols[i])) : 0.f;
          const float p1 = ((vis >> (i + 1)) & 1u) ? ex2(fmaf(__uint_as_float(sv[i + 1]), p.sl2, -cols[i + 1])) : 0.f;
          pf[i] = p0;
          pf[i + 1] = p1;
          if constexpr (P8)
            pp[i / 2] = e4m3_round_bf16x2(p0, p1);
          else
            pp[i / 2] = pack_bf16(p0, p1);
        }
      }
      // P^T words (bf16x2; P8: e4m3-rounded) of chunk c go to columns
      // [16c, 16c + 16), scores another warp of this quarter reads: store
      // them once every compute thread holds its chunk
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->s_read));
      ok = wait_bar(smem_u32(&bars->s_read), t & 1, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      tmem_st16(tbase + lane_off + T_S + c * 16, pp);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->p_full));
      // phase 2: dS^T = P^T o (dP^T - Dr)
      ok = wait_bar(smem_u32(&bars->dp_full), t & 1, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t pd[16];
      {
        uint32_t dp[32];
        tmem_ld32(tbase + lane_off + T_DP + c * 32, dp);
        tmem_ld_wait(dp);
#pragma unroll
        for (int i = 0; i < 32; i += 2)
          pd[i / 2] = pack_bf16(pf[i] * (__uint_as_float(dp[i]) - cols[32 + i]),
                                pf[i + 1] * (__uint_as_float(dp[i + 1]) - cols[33 + i]));
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->dp_read));
      ok = wait_bar(smem_u32(&bars->dp_read), t & 1, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      tmem_st16(tbase + lane_off + T_DP + c * 16, pd);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->ds_full));
    }
    if (ok) {
      ok = wait_bar(smem_u32(&bars->acc_full), 0, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const bool w = key < p.Nkv;
      // units of 32 accumulator columns: dV chunks, then dK chunks; four warps per quarter share them
      for (int u = c; u < 2 * (D / 32); u += 4) {
        const bool is_dv = u < D / 32;
        const int cc = is_dv ? u : u - D / 32;
        uint16_t* dst = (is_dv ? p.dv : p.dk) + ((size_t)bh * p.Nkv + key) * D + cc * 32;
        if (nit > 0) {
          bwd_store_chunk(tbase + lane_off + (is_dv ? T_DV : T_DK) + cc * 32, dst, is_dv ? 1.f : p.scale, w);
        } else if (w) {  // no query sees these keys
#pragma unroll
          for (int e = 0; e < 32; e += 8) *reinterpret_cast<uint4*>(dst + e) = make_uint4(0, 0, 0, 0);
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
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
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
    mbar_init(smem_u32(&bars->dp_full), 1);
    mbar_init(smem_u32(&bars->p_full), C::CT);
    mbar_init(smem_u32(&bars->ds_full), C::CT);
    mbar_init(smem_u32(&bars->s_read), C::CT);
    mbar_init(smem_u32(&bars->dp_read), C::CT);
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
  // TMEM: S [0,128), dP [128,256), dQ [256, 256+D), dS (bf16x2) [384, 448):
  // dS has columns of its own, so no compute warp writes over scores another reads
  const uint32_t T_S = 0, T_DP = 128, T_DQ = 256, T_DS = 384;

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
      auto stage = [&](int t) { return sbase + C::ST_OFF + (t % C::NST) * C::STAGE; };
      auto stage_full = [&](int t) -> bool {
        const bool r = wait_bar(smem_u32(&bars->st_full[t % C::NST]), (t / C::NST) & 1, abort_flag, p.timeout_ns);
        tc_fence_after();
        return r;
      };
      // S(0) = Q K_0^T, dP(0) = dO V_0^T
      if (ok && nj > 0 && (ok = stage_full(0))) {
        bwd_issue_score<D>(tbase + T_S, dQ, smem_desc(stage(0), 16, 1024));
        tc_commit(smem_u32(&bars->s_full));
        bwd_issue_score<D>(tbase + T_DP, dDO, smem_desc(stage(0) + C::TILE, 16, 1024));
        tc_commit(smem_u32(&bars->dp_full));
      }
      for (int t = 0; t < nj && ok; ++t) {
        if (t + 1 < nj) {  // S(t+1) once the compute warps hold S(t) in registers
          ok = wait_bar(smem_u32(&bars->p_full), t & 1, abort_flag, p.timeout_ns);
          if (!ok || !(ok = stage_full(t + 1))) break;
          bwd_issue_score<D>(tbase + T_S, dQ, smem_desc(stage(t + 1), 16, 1024));
          tc_commit(smem_u32(&bars->s_full));
        }
        ok = wait_bar(smem_u32(&bars->ds_full), t & 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        // dQ += dS K_t (K_t rows are the contraction: B MN-major)
        bwd_issue_acc<D>(tbase + T_DQ, tbase + T_DS, smem_desc(stage(t), C::HALF, 1024), t > 0);
        tc_commit(smem_u32(&bars->st_empty[t % C::NST]));
        if (t + 1 < nj) {  // dP(t+1) once the compute warps hold dP(t) (ds_full)
          bwd_issue_score<D>(tbase + T_DP, dDO, smem_desc(stage(t + 1) + C::TILE, 16, 1024));
          tc_commit(smem_u32(&bars->dp_full));
        }
      }
      if (ok) tc_commit(smem_u32(&bars->acc_full));
      if (!ok) {
        tc_commit(smem_u32(&bars->drain));
        wait_bar_drain(smem_u32(&bars->drain), 0, p.timeout_ns);
      }
    }
    __syncwarp();
  } else {
    // compute warp: TMEM lane quarter warp % 4 (its query rows), key columns [32c, 32c + 32)
    const int cw = warp - 2;
    const int quarter = warp & 3, c = cw >> 2;
    const int rr = quarter * 32 + lane;
    const int row = q0 + rr;  // this thread's query row
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const bool live = row < p.Nq;
    const float lse2 = live ? p.lse[(size_t)bh * p.Nq + row] * 1.4426950408889634f : INFINITY;
    const float rd = live ? p.rowdot[(size_t)bh * p.Nq + row] : 0.f;
    bool ok = true;
    for (int t = 0; t < nj && ok; ++t) {
      const int kc = t * 128 + 32 * c;  // first key column of this chunk
      ok = wait_bar(smem_u32(&bars->s_full), t & 1, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // phase 1: P = exp2(S sl2 - lse2) (masked) into fp32 registers; then
      // the S columns are free for S(t+1)
      float pf[32];
      {
        uint32_t sv[32];
        tmem_ld32(tbase + lane_off + T_S + c * 32, sv);
        tmem_ld_wait(sv);
        // visible keys: k < Nkv and (causal) k <= row + off
        int hi = p.Nkv - kc;
        if (p.causal) hi = min(hi, row + off - kc + 1);
        if (!live) hi = 0;
        const uint32_t vis = bwd_mask32(0, hi);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          pf[i] = ((vis >> i) & 1u) ? ex2(fmaf(__uint_as_float(sv[i]), p.sl2, -lse2)) : 0.f;
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->p_full));
      // phase 2: dS = P o (dP - Dr), bf16 into this chunk's dS columns
      ok = wait_bar(smem_u32(&bars->dp_full), t & 1, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t pd[16];
      {
        uint32_t dp[32];
        tmem_ld32(tbase + lane_off + T_DP + c * 32, dp);
        tmem_ld_wait(dp);
#pragma unroll
        for (int i = 0; i < 32; i += 2)
          pd[i / 2] = pack_bf16(pf[i] * (__uint_as_float(dp[i]) - rd), pf[i + 1] * (__uint_as_float(dp[i + 1]) - rd));
      }
      tmem_st16(tbase + lane_off + T_DS + c * 16, pd);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->ds_full));
    }
    if (ok) {
      ok = wait_bar(smem_u32(&bars->acc_full), 0, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      uint16_t* dst = p.dq + ((size_t)bh * p.Nq + row) * D;
      for (int cc = c; cc < D / 32; cc += 4) {
        if (nj > 0) {
          bwd_store_chunk(tbase + lane_off + T_DQ + cc * 32, dst + cc * 32, p.scale, live);
        } else if (live) {  // no key visible to this tile
#pragma unroll
          for (int e = 0; e < 32; e += 8) *reinterpret_cast<uint4*>(dst + cc * 32 + e) = make_uint4(0, 0, 0, 0);
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

}  // namespace ta
