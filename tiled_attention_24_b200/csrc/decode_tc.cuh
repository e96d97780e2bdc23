// Grouped-query decode on the tensor cores (d = 128).
//
// With grouped-query attention several query heads share one cached key /
// value head ("FlashAttention 4: fast, memory-saving attention for LLMs",
// compatibility and current status: GQA / MQA), so one pass over a cache
// head serves a small matrix of queries: decode becomes a thin GEMM.  One CTA
// takes G <= 8 query heads of one cache head and one chunk of its keys:
//
//   S  = Q K_j^T   tcgen05.mma kind::f16, M = 128, N = 64 keys, K = d
//   softmax of the G rows (one thread per query head, lazy rescale tau = 8)
//   O += P V_j     tcgen05.mma kind::f16, M = 128, N = d, K = 64 keys
//
// The G query rows are the A operand of both MMAs: a single 8-row, 128-byte
// swizzle atom per 64 columns, read with a zero stride between 8-row groups
// (SBO = 0), so the MMA's 128 rows are 16 copies of rows 0-7 and Q and P take
// 1 KB per 64 columns of shared memory.  Rows G..7 of P are zero; S and O rows
// other than 0..G-1 are never read.  The tensor cores do ~2x128x64x128 FLOPs
// per 32 KB key/value tile -- far below their rate -- so the kernel streams
// the cache at HBM speed: a TMA producer keeps NSTAGE tiles in flight, two
// CTAs share an SM (256 TMEM columns and ~104 KB of shared memory each), and
// each CTA is persistent: it walks the (head group, chunk) items with a
// stride of the grid, and its ring, barriers and tensor memory carry over
// from one item to the next, so the cache stream does not stop between items
// (a CTA per item cost ~2.4 us of set-up and drain each).  Q is double-
// buffered per item; the one O accumulator is read out by the epilogue before
// the next item's first P V overwrites it.
//
// Warps: 0 = softmax + epilogue (its TMEM lane quarter holds rows 0-31),
// 1 = TMA producer, 2 = MMA issuer, 3 = TMEM allocation.  Results are the
// normalised partial O_c and LSE_c of the split-KV scheme, merged by
// decode_combine_kernel.  Every wait is bounded (wait_bar).
#pragma once
#include "ptx.cuh"
#include "fwd_bf16.cuh"  // wait_bar_drain

namespace ta {

struct DecTcCfg {
  static constexpr int D = 128, KT = 64;        // head dim, keys per tile
  static constexpr int NSTAGE = 3;
  static constexpr int BOX = KT * 128;          // one 64-column block of a K or V tile (8 KB)
  static constexpr int KV_TILE = 2 * BOX;       // K or V tile, 128 d x 64 keys (16 KB)
  static constexpr int STAGE = 2 * KV_TILE;     // K then V (32 KB)
  static constexpr int Q_OFF = NSTAGE * STAGE;  // Q: two buffers of two 1 KB atoms (d 0-63, 64-127)
  static constexpr int P_OFF = Q_OFF + 4096;    // P: two buffers of one 1 KB atom
  static constexpr int BAR_OFF = P_OFF + 2048;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;  // + alignment slack
  static constexpr int THREADS = 128;
  static constexpr uint32_t T_S = 0, T_O = 128;  // TMEM: S_0, S_1 [0,128), O [128,256)
  static constexpr uint32_t ID_S = idesc_bf16_f32(128, KT, false);
  static constexpr uint32_t ID_PV = idesc_bf16_f32(128, D, true);
  static constexpr float TAU = 8.0f;
};

struct DecTcBars {
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t kv_full[DecTcCfg::NSTAGE];
  uint64_t kv_empty[DecTcCfg::NSTAGE];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint64_t o_full;
  uint64_t o_free;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(DecTcBars) <= 256, "barrier block too large");

// One work item: G query heads (rows bh0..bh0+G-1 of the query matrix) of
// cache head kvh against keys [key0, key0 + nk) of chunk c.
struct DecTcItem {
  int bh0, kvh, c, nk, nt;
  long long key0;
};
template <int G>
__device__ __forceinline__ DecTcItem dec_tc_item(int it, int S, int chunk, int Nkv, int group, int Hq,
                                                 const int* __restrict__ seqlens) {
  DecTcItem r;
  r.bh0 = (it / S) * G;
  r.c = it % S;
  r.kvh = r.bh0 / group;  // G divides the group
  const int len = seqlens ? min(max(seqlens[r.bh0 / Hq], 0), Nkv) : Nkv;
  const int ch = seqlens ? (len + S - 1) / S : chunk;
  r.key0 = (long long)r.c * ch;
  r.nk = (int)max(0LL, min((long long)len, r.key0 + ch) - r.key0);
  r.nt = (r.nk + DecTcCfg::KT - 1) / DecTcCfg::KT;
  return r;
}

// tmK / tmV: the cache [B*Hkv][Nkv][128] as (128, Nkv, B*Hkv), boxes 64 x 64 x 1;
// tmQ: the queries [B*Hq][128] as (128, B*Hq), boxes 64 x 8 (rows past the
// item's G heads are loaded but never used).  n_items = (B*Hq / G) * S.
template <int G>
__global__ void __launch_bounds__(DecTcCfg::THREADS, 2)
    decode_gqa_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, float* __restrict__ o_part,
                         float* __restrict__ lse_part, int n_items, int Nkv, int S, int chunk, float sl2,
                         int group, const int* __restrict__ seqlens, int Hq, unsigned long long timeout_ns) {
  using C = DecTcCfg;
  static_assert(G >= 1 && G <= 8, "at most 8 query heads per CTA");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  DecTcBars* bars = reinterpret_cast<DecTcBars*>(smem + C::BAR_OFF);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->q_full[b]), 1);
      mbar_init(smem_u32(&bars->q_empty[b]), 1);
      mbar_init(smem_u32(&bars->s_full[b]), 1);
      mbar_init(smem_u32(&bars->s_free[b]), 1);
      mbar_init(smem_u32(&bars->p_full[b]), 1);
      mbar_init(smem_u32(&bars->pv_done[b]), 1);
    }
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(smem_u32(&bars->kv_full[s]), 1);
      mbar_init(smem_u32(&bars->kv_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->o_full), 1);
    mbar_init(smem_u32(&bars->o_free), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 3) {
    tmem_alloc(smem_u32(&bars->tmem_base), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;

  if (warp == 1) {
    // ================================================================ producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      bool ok = true;
      int g = 0, qi = 0;  // tiles and items (with keys) loaded so far
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const DecTcItem I = dec_tc_item<G>(it, S, chunk, Nkv, group, Hq, seqlens);
        if (I.nt == 0) continue;
        const int qb = qi & 1;
        // Q buffer qb was last read by the S MMAs of item qi - 2
        if (qi >= 2 && !(ok = wait_bar(smem_u32(&bars->q_empty[qb]), ((qi - 2) >> 1) & 1, abort_flag, timeout_ns)))
          break;
        const uint32_t qbar = smem_u32(&bars->q_full[qb]);
        mbar_arrive_expect_tx(qbar, 2048);
        tma_load_2d(sbase + C::Q_OFF + qb * 2048, &tmQ, qbar, 0, I.bh0);
        tma_load_2d(sbase + C::Q_OFF + qb * 2048 + 1024, &tmQ, qbar, 64, I.bh0);
        ++qi;
        for (int t = 0; t < I.nt; ++t, ++g) {
          const int st = g % C::NSTAGE;
          ok = wait_bar(smem_u32(&bars->kv_empty[st]), ((g / C::NSTAGE) & 1) ^ 1, abort_flag, timeout_ns);
          if (!ok) break;
          const uint32_t fb = smem_u32(&bars->kv_full[st]);
          mbar_arrive_expect_tx(fb, C::STAGE);
          const uint32_t dst = sbase + st * C::STAGE;
          const int key = (int)(I.key0 + (long long)t * C::KT);
          tma_load_3d(dst, &tmK, fb, 0, key, I.kvh);
          tma_load_3d(dst + C::BOX, &tmK, fb, 64, key, I.kvh);
          tma_load_3d(dst + C::KV_TILE, &tmV, fb, 0, key, I.kvh);
          tma_load_3d(dst + C::KV_TILE + C::BOX, &tmV, fb, 64, key, I.kvh);
        }
      }
      // never leave a copy in flight (after a normal run these have all completed)
      for (int back = 1; back <= 2 && qi - back >= 0; ++back)
        wait_bar_drain(smem_u32(&bars->q_full[(qi - back) & 1]), ((qi - back) >> 1) & 1, timeout_ns);
      for (int back = 1; back <= C::NSTAGE && g - back >= 0; ++back) {
        const int i2 = g - back;
        wait_bar_drain(smem_u32(&bars->kv_full[i2 % C::NSTAGE]), (i2 / C::NSTAGE) & 1, timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      bool ok = true;
      int g = 0, qi = 0;
      // P V of global tile i (stage i % NSTAGE, P buffer i & 1); `first`: the
      // item's first tile, which overwrites O once the epilogue has read it
      auto issue_PV = [&](int i, bool first, int item) -> bool {
        const int b = i & 1, st = i % C::NSTAGE;
        if (first && item > 0) {
          if (!spin_bar(smem_u32(&bars->o_free), (item - 1) & 1, abort_flag, timeout_ns)) return false;
        }
        if (!spin_bar(smem_u32(&bars->p_full[b]), (i >> 1) & 1, abort_flag, timeout_ns)) return false;
        tc_fence_after();
        const uint64_t dP = smem_desc(sbase + C::P_OFF + b * 1024, 16, 0);
        const uint64_t dV = smem_desc(sbase + st * C::STAGE + C::KV_TILE, C::BOX, 1024);
#pragma unroll
        for (int kk = 0; kk < C::KT / 16; ++kk)
          mma_f16_ss(tbase + C::T_O, dP + (uint64_t)((kk * 32) >> 4), dV + (uint64_t)((kk * 2048) >> 4), C::ID_PV,
                     (!first || kk > 0) ? 1u : 0u);
        tc_commit(smem_u32(&bars->pv_done[b]));
        tc_commit(smem_u32(&bars->kv_empty[st]));
        return true;
      };
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const DecTcItem I = dec_tc_item<G>(it, S, chunk, Nkv, group, Hq, seqlens);
        if (I.nt == 0) continue;
        const int qb = qi & 1;
        if (!(ok = spin_bar(smem_u32(&bars->q_full[qb]), (qi >> 1) & 1, abort_flag, timeout_ns))) break;
        const uint64_t dQ = smem_desc(sbase + C::Q_OFF + qb * 2048, 16, 0);
        for (int t = 0; t < I.nt && ok; ++t, ++g) {
          const int st = g % C::NSTAGE, b = g & 1;
          if (!(ok = spin_bar(smem_u32(&bars->kv_full[st]), (g / C::NSTAGE) & 1, abort_flag, timeout_ns))) break;
          if (g >= 2) {  // the softmax has read S(g-2) from this buffer
            if (!(ok = spin_bar(smem_u32(&bars->s_free[b]), ((g - 2) >> 1) & 1, abort_flag, timeout_ns))) break;
            tc_fence_after();
          }
          const uint64_t dK = smem_desc(sbase + st * C::STAGE, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < C::D / 16; ++kk) {
            const uint64_t offq = (uint64_t)(((kk >> 2) * 1024 + (kk & 3) * 32) >> 4);
            const uint64_t offk = (uint64_t)(((kk >> 2) * C::BOX + (kk & 3) * 32) >> 4);
            mma_f16_ss(tbase + C::T_S + b * C::KT, dQ + offq, dK + offk, C::ID_S, kk > 0);
          }
          tc_commit(smem_u32(&bars->s_full[b]));
          if (t == I.nt - 1) tc_commit(smem_u32(&bars->q_empty[qb]));
          if (t >= 1) ok = issue_PV(g - 1, t == 1, qi);
        }
        if (ok) ok = issue_PV(g - 1, I.nt == 1, qi);
        if (ok) tc_commit(smem_u32(&bars->o_full));
        ++qi;
      }
      if (!ok) {  // every MMA issued so far must finish before TMEM is freed
        tc_commit(smem_u32(&bars->drain));
        wait_bar_drain(smem_u32(&bars->drain), 0, timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 0) {
    // ================================================================ softmax (thread = query head)
    const int row = lane;  // TMEM lane == MMA row; rows < G are the item's heads
    bool ok = true;
    int g = 0, qi = 0;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      const DecTcItem I = dec_tc_item<G>(it, S, chunk, Nkv, group, Hq, seqlens);
      if (I.nt == 0) {  // no keys in this chunk: O_c = 0, LSE_c = -inf
        if (row < G) {
          float4* dst = reinterpret_cast<float4*>(o_part + ((size_t)(I.bh0 + row) * S + I.c) * C::D);
#pragma unroll 4
          for (int i = 0; i < C::D / 4; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          lse_part[(size_t)(I.bh0 + row) * S + I.c] = -INFINITY;
        }
        continue;
      }
      float m_ref = -INFINITY, l = 0.f;
      for (int t = 0; t < I.nt; ++t, ++g) {
        const int b = g & 1;
        ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&bars->s_full[b]), (g >> 1) & 1, abort_flag, timeout_ns));
        if (!ok) break;
        tc_fence_after();
        uint32_t s[2][32];
        tmem_ld32(tbase + C::T_S + b * C::KT, s[0]);
        tmem_ld32(tbase + C::T_S + b * C::KT + 32, s[1]);
        tmem_ld_wait(s[0]);
        tmem_ld_wait(s[1]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->s_free[b]));
        const int lim = I.nk - t * C::KT;  // keys [lim, 64) of this tile lie past the chunk
        if (lim < C::KT) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (h * 32 + i >= lim) s[h][i] = 0xFF800000u;  // -inf
        }
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          mx0 = fmax3(mx0, __uint_as_float(s[0][i]), __uint_as_float(s[0][i + 1]));
          mx1 = fmax3(mx1, __uint_as_float(s[1][i]), __uint_as_float(s[1][i + 1]));
        }
        const float m_blk = fmaxf(mx0, mx1) * sl2;
        const bool need = row < G && m_blk > m_ref + C::TAU;
        float factor = 1.f;
        if (need) {
          factor = ex2(m_ref - m_blk);  // 0 when m_ref == -inf
          l *= factor;
          m_ref = m_blk;
        }
        if (t > 0 && __any_sync(0xffffffffu, need)) {
          // O must hold P V(g-1) before it is scaled
          ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&bars->pv_done[(g - 1) & 1]), ((g - 1) >> 1) & 1,
                                                abort_flag, timeout_ns));
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < C::D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tbase + C::T_O + cc * 32, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
            tmem_st32(tbase + C::T_O + cc * 32, o);
          }
          tmem_st_wait();
        }
        // P(g) goes to buffer b, which P V(g-2) read
        if (g >= 2) {
          ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&bars->pv_done[b]), ((g - 2) >> 1) & 1, abort_flag,
                                                timeout_ns));
          if (!ok) break;
        }
        const float mr = (m_ref == -INFINITY) ? 0.f : m_ref;
        const uint64_t nm = f2(-mr, -mr), sc = f2(sl2, sl2);
        uint32_t w[32];
        float ls = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float x0, x1;
            f2_split(ffma2(f2(__uint_as_float(s[h][i]), __uint_as_float(s[h][i + 1])), sc, nm), x0, x1);
            const float p0 = ex2(x0), p1 = ex2(x1);
            ls += p0 + p1;
            w[h * 16 + i / 2] = pack_bf16(p0, p1);
          }
        if (row < G) l += ls;
        if (row < 8) {
          uint8_t* prow = smem + C::P_OFF + b * 1024 + row * 128;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 v = (row < G) ? make_uint4(w[4 * ch], w[4 * ch + 1], w[4 * ch + 2], w[4 * ch + 3])
                                      : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(prow + ((ch ^ row) << 4)) = v;
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[b]));
      }
      if (!ok) break;
      // ---- epilogue of the item: O / l and LSE for rows 0..G-1, then O is free
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&bars->o_full), qi & 1, abort_flag, timeout_ns));
      if (!ok) break;
      tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      float* dst = o_part + ((size_t)(I.bh0 + row) * S + I.c) * C::D;
#pragma unroll 1
      for (int cc = 0; cc < C::D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tbase + C::T_O + cc * 32, o);
        tmem_ld_wait(o);
        if (row < G) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + cc * 32 + i) =
                make_float4(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                            __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->o_free));
      if (row < G)
        lse_part[(size_t)(I.bh0 + row) * S + I.c] = (l > 0.f) ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
      ++qi;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 3) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

}  // namespace ta
