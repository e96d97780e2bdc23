// FP8 (e4m3) tiled attention forward for sm_100a: tcgen05 kind::f8f6f4.
//
// "Can a full-day context beat one minute? Flash attention and the
// sequence-length question", FA3 list item 3: FP8 runs the matmuls at twice
// the 16-bit rate; outliers break naive FP8 attention, so Q and K are rotated
// (randomised Hadamard, see the FP8 quantisers) before the quantisation.
// Operands: e4m3 codes with one fp32 scale per Q / K token row and one per V
// channel.  Steps per 128-key block j (tiling, masking, online softmax as the
// bf16 kernel):
//   S  = codes(Q) codes(K_j)^T                 fp32 in TMEM
//   x  = S * s_Q[row] * s_K[key] * scale * log2(e) / rot_d     (rot_d = d when
//        Q and K were rotated: the rotation multiplies Q K^T by d)
//   P~ = e4m3_rne(2^(x - m))   (unit scale),   l += sum P~ (by the tensor
//        core: P~ times a 128 x 16 matrix of ones, into TMEM)
//   m: lazy reference max ("FlashAttention 4" page, smarter online softmax
//        rescaling): it moves to the block max only when that exceeds it by
//        more than TAU = 8, so P~ <= 2^8 = 256 stays inside e4m3's range (448)
//   O += P~ codes(V_j)                          fp32 in TMEM, corrected in
//        place by 2^(m_old - m) when the max grows
//   O_c = O_c * s_V[c] / l (fp32 output), LSE = ln2 * (m + log2 l).
//
// CTA = one (batch, head) x two 128-row query tiles; warps: 0 TMA producer,
// 1 MMA issuer, 2-3 idle (registers given to the softmax warps), 4-7 and 8-11
// softmax / correction / epilogue of tiles 0 and 1 (thread = row).  One TMEM
// score buffer shared by the tiles (moved to registers at once, then released
// to the other tile), O_0 [128,256), O_1 [256,384), P~ of tile t (A operand
// of P V, 128 keys = 32 columns) [384 + 32 t, +32), row sums l_t
// [448 + 16 t, +16) (column 0 read).  One P~ buffer per tile: the softmax
// waits for P V_t(j-1) before it stores P~_t(j) (its exps are already in
// registers by then).  MMA order as the FP4 kernel: S_0(0), S_1(0), S_0(1),
// then per block P V_0(j), S_1(j+1), P V_1(j), S_0(j+2).  Shared memory: Q
// tiles and a ring of K / V tiles (128 x 128 bytes, 128-byte swizzle), the
// ones matrix, per-warp key constants.  d = 128 only.
#pragma once
#include "ptx.cuh"
#include "fwd_bf16.cuh"  // fwd_tile_kv_count, wait_bar_drain

namespace ta {

struct FwdF8Params {
  const float* q_scale;  // [BH][Nq]
  const float* k_scale;  // [BH][Nkv]
  const float* v_scale;  // [BH][128] per channel
  float* o;              // [BH][Nq][128] fp32
  float* lse;            // [BH][Nq]
  int Nq, Nkv, n_qp, Tc;
  int causal;
  int ks_vec;  // k_scale rows 16-byte aligned: vector loads
  float sl2;   // scale * log2(e) / rot_d
  unsigned long long timeout_ns;
};

// kind::f8f6f4 instruction descriptor: D = f32 (1), A = B = e4m3 (0),
// M = 128; b_mn: B stored MN-major.
__host__ __device__ constexpr uint32_t idesc_f8(int N, bool b_mn) {
  return (1u << 4) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

struct FwdF8Cfg {
  static constexpr int TILE = 128 * 128;  // 128 rows x 128 e4m3 codes
  static constexpr int NSLOT = 8;
  static constexpr int Q_OFF = 0;                         // Q_0, Q_1
  static constexpr int SLOT_OFF = 2 * TILE;
  static constexpr int ONES_OFF = SLOT_OFF + NSLOT * TILE;  // 16 x 128 e4m3 ones (0x38)
  static constexpr int KC_OFF = ONES_OFF + 2048;            // [8 warps][2 bufs][128] floats
  static constexpr int BAR_OFF = KC_OFF + 8 * 2 * 128 * 4;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
  static constexpr int THREADS = 384;
  // register split (launch: 384 threads x 168): warpgroup 0 drops to 72, the
  // two softmax warpgroups rise to 216: 128*72 + 256*216 = 64512 = 384*168
  static constexpr int REG_LOW = 72, REG_HIGH = 216;
  static constexpr float TAU = 8.f;  // lazy-rescale threshold (log2 units)
  static constexpr uint32_t ID_S = idesc_f8(128, false);
  static constexpr uint32_t ID_PV = idesc_f8(128, true);  // V is MN-major
  static constexpr uint32_t ID_L = idesc_f8(16, false);   // P~ x ones: row sums
  static constexpr uint32_t T_S = 0, T_O = 128, T_P8 = 384, T_L = 448;
};

struct FwdF8Bars {
  uint64_t q_full;
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint64_t s_full[2];     // MMA -> softmax of tile t: S_t(j) in the score buffer
  uint64_t s_free;        // softmax -> MMA: the score buffer's scores are in registers
  uint64_t p_full[2][2];  // [tile][j % 2]: P~_t(j) in TMEM, O_t and l_t corrected
  uint64_t pv_done[2];    // [tile]: P V_t(j) finished
  uint64_t o_full[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(FwdF8Bars) <= 256, "barrier block too large");

__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ uint32_t e4m3x2_pair(float lo, float hi) {  // non-negative inputs
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(384, 1)
    fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdF8Params p) {
  using C = FwdF8Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FwdF8Bars* bars = reinterpret_cast<FwdF8Bars*>(smem + C::BAR_OFF);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: (batch*head, pair of query tiles); heaviest pairs first when causal
  const int BH = gridDim.x / p.n_qp;
  const int bh = p.causal ? (int)(blockIdx.x % BH) : (int)(blockIdx.x / p.n_qp);
  const int qp = p.causal ? p.n_qp - 1 - (int)(blockIdx.x / BH) : (int)(blockIdx.x % p.n_qp);
  int r0[2], n[2];
  bool present[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    r0[t] = qp * 256 + t * 128;
    present[t] = r0[t] < p.Nq;
    n[t] = fwd_tile_kv_count(r0[t], p.Nq, p.Nkv, p.Tc, p.causal);
  }
  const int nmax = max(n[0], n[1]);
  volatile int* abort_flag = &bars->abort;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(smem_u32(&bars->kv_full[s]), 1);
      mbar_init(smem_u32(&bars->kv_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->s_free), 128);
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&bars->s_full[t]), 1);
      mbar_init(smem_u32(&bars->p_full[t][0]), 128);
      mbar_init(smem_u32(&bars->p_full[t][1]), 128);
      mbar_init(smem_u32(&bars->pv_done[t]), 1);
      mbar_init(smem_u32(&bars->o_full[t]), 1);
    }
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  // constant B operand of the row-sum MMA: e4m3 ones (every byte 0x38, so the
  // swizzle does not matter)
  for (int i = threadIdx.x; i < 2048 / 16; i += C::THREADS)
    *reinterpret_cast<uint4*>(smem + C::ONES_OFF + i * 16) = make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;

  if (warp < 4) {
   reg_dealloc<C::REG_LOW>();
   if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const uint32_t qbar = smem_u32(&bars->q_full);
      mbar_arrive_expect_tx(qbar, (present[0] + present[1]) * C::TILE);
      for (int t = 0; t < 2; ++t)
        if (present[t]) tma_load_3d(sbase + C::Q_OFF + t * C::TILE, &tmQ, qbar, 0, r0[t], bh);
      int it = 0;
      bool ok = true;
      for (int j = 0; j < nmax && ok; ++j) {
        for (int w = 0; w < 2 && ok; ++w, ++it) {
          const int slot = it % C::NSLOT;
          ok = wait_bar(smem_u32(&bars->kv_empty[slot]), ((it / C::NSLOT) & 1) ^ 1, abort_flag, p.timeout_ns);
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
      const uint64_t dQ0 = smem_desc(sbase + C::Q_OFF, 16, 1024);
      const uint64_t dK0 = smem_desc(sbase + C::SLOT_OFF, 16, 1024);
      const uint64_t dV0 = smem_desc(sbase + C::SLOT_OFF, C::TILE, 1024);
      const uint64_t dOnes = smem_desc(sbase + C::ONES_OFF, 16, 1024);
      int n_s = 0;  // S MMAs issued so far (the score buffer's uses)
      auto issue_S = [&](int t, int j) -> bool {
        if (n_s > 0) {
          if (!wait_bar(smem_u32(&bars->s_free), (n_s - 1) & 1, abort_flag, p.timeout_ns)) return false;
          tc_fence_after();
        }
        const int it = 2 * j, s = it % C::NSLOT;
        const bool first = (t == 0) || (j >= n[0]);
        const bool last = (t == 1) || (j >= n[1]);
        if (first) {
          if (!wait_bar(smem_u32(&bars->kv_full[s]), (it / C::NSLOT) & 1, abort_flag, p.timeout_ns)) return false;
          tc_fence_after();
        }
        const uint64_t dq = dQ0 + (uint64_t)(t * (C::TILE >> 4));
        const uint64_t dk = dK0 + (uint64_t)(s * (C::TILE >> 4));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = 32 e4m3 per MMA
          mma_f8_ss(tbase + C::T_S, dq + (uint64_t)(kk * 2), dk + (uint64_t)(kk * 2), C::ID_S, kk > 0);
        tc_commit(smem_u32(&bars->s_full[t]));
        if (last) tc_commit(smem_u32(&bars->kv_empty[s]));
        ++n_s;
        return true;
      };
      auto issue_PV = [&](int t, int j) -> bool {
        const int it = 2 * j + 1, s = it % C::NSLOT;
        const bool first = (t == 0) || (j >= n[0]);
        const bool last = (t == 1) || (j >= n[1]);
        if (first) {
          if (!wait_bar(smem_u32(&bars->kv_full[s]), (it / C::NSLOT) & 1, abort_flag, p.timeout_ns)) return false;
        }
        if (!wait_bar(smem_u32(&bars->p_full[t][j & 1]), (j >> 1) & 1, abort_flag, p.timeout_ns)) return false;
        tc_fence_after();
        const uint64_t dv = dV0 + (uint64_t)(s * (C::TILE >> 4));
        const uint32_t aP = tbase + C::T_P8 + 32 * t;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 32 keys per MMA: 8 P~ columns / 32 rows x 128 B of V
          mma_f8_ts(tbase + C::T_O + 128 * t, aP + kk * 8, dv + (uint64_t)(kk * (4096 >> 4)), C::ID_PV,
                    (j > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // l_t += P~ 1
          mma_f8_ts(tbase + C::T_L + 16 * t, aP + kk * 8, dOnes + (uint64_t)(kk * 2), C::ID_L,
                    (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(smem_u32(&bars->pv_done[t]));
        if (last) tc_commit(smem_u32(&bars->kv_empty[s]));
        if (j == n[t] - 1) tc_commit(smem_u32(&bars->o_full[t]));
        return true;
      };
      if (ok) {
        for (int t = 0; t < 2; ++t)
          if (present[t] && n[t] == 0) tc_commit(smem_u32(&bars->o_full[t]));
      }
      if (ok && n[0] > 0) ok = issue_S(0, 0);
      if (ok && n[1] > 0) ok = issue_S(1, 0);
      if (ok && n[0] > 1) ok = issue_S(0, 1);
      for (int j = 0; j < nmax && ok; ++j) {
        if (j < n[0] && !(ok = issue_PV(0, j))) break;
        if (j + 1 < n[1] && !(ok = issue_S(1, j + 1))) break;
        if (j < n[1] && !(ok = issue_PV(1, j))) break;
        if (j + 2 < n[0] && !(ok = issue_S(0, j + 2))) break;
      }
      if (!ok) {
        tc_commit(smem_u32(&bars->drain));
        wait_bar_drain(smem_u32(&bars->drain), 0, p.timeout_ns);
      }
    }
    __syncwarp();
   }
  } else {
    reg_alloc<C::REG_HIGH>();
    // ================================================================ softmax
    const int t = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int rr = quarter * 32 + lane;
    const int row = r0[t] + rr;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tbase + lane_off + C::T_S;
    const uint32_t tO = tbase + lane_off + C::T_O + 128 * t;
    const uint32_t tL = tbase + lane_off + C::T_L + 16 * t;
    const int off = p.Nkv - p.Nq;
    const float qs_row = (present[t] && row < p.Nq) ? p.q_scale[(size_t)bh * p.Nq + row] : 0.f;
    const float* ksrow = p.k_scale + (size_t)bh * p.Nkv;
    // Per-column constants of a key block, kc = s_K * scale * log2(e) / rot_d,
    // in this warp's own shared buffer; lane l stages columns [4l, 4l + 4),
    // the next block's scales loaded one block ahead.
    float* kcbuf = reinterpret_cast<float*>(smem + C::KC_OFF) + (warp - 4) * (2 * 128);
    float4 ks_next = make_float4(0.f, 0.f, 0.f, 0.f);
    auto load_ks = [&](int jj) {
      const int c0 = jj * 128 + lane * 4;
      if (p.ks_vec && c0 + 3 < p.Nkv) {
        ks_next = __ldg(reinterpret_cast<const float4*>(ksrow + c0));
      } else {
        ks_next.x = (c0 + 0 < p.Nkv) ? ksrow[c0 + 0] : 0.f;
        ks_next.y = (c0 + 1 < p.Nkv) ? ksrow[c0 + 1] : 0.f;
        ks_next.z = (c0 + 2 < p.Nkv) ? ksrow[c0 + 2] : 0.f;
        ks_next.w = (c0 + 3 < p.Nkv) ? ksrow[c0 + 3] : 0.f;
      }
    };
    auto stage_ks = [&](int jj) {
      *reinterpret_cast<float4*>(kcbuf + (jj & 1) * 128 + lane * 4) =
          make_float4(ks_next.x * p.sl2, ks_next.y * p.sl2, ks_next.z * p.sl2, ks_next.w * p.sl2);
    };
    float m_ref = -INFINITY;  // l lives in TMEM (column tL), summed by the tensor core
    bool ok = present[t];
    if (ok && n[t] > 0) {
      load_ks(0);
      stage_ks(0);
      if (n[t] > 1) load_ks(1);
      __syncwarp();
    }
    for (int j = 0; j < n[t] && ok; ++j) {
      const int kb = j * 128;
      ok = wait_bar(smem_u32(&bars->s_full[t]), j & 1, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t s[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, s[c]);
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_wait(s[c]);
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->s_free));  // the score buffer goes to the other tile
      // y = S * kc (= x / s_Q), masked
      const float* kcb = kcbuf + (j & 1) * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 kc = *reinterpret_cast<const float4*>(kcb + c * 32 + i);
          float a0, a1, a2, a3;
          f2_split(fmul2(f2(__uint_as_float(s[c][i]), __uint_as_float(s[c][i + 1])), f2(kc.x, kc.y)), a0, a1);
          f2_split(fmul2(f2(__uint_as_float(s[c][i + 2]), __uint_as_float(s[c][i + 3])), f2(kc.z, kc.w)), a2, a3);
          s[c][i] = __float_as_uint(a0);
          s[c][i + 1] = __float_as_uint(a1);
          s[c][i + 2] = __float_as_uint(a2);
          s[c][i + 3] = __float_as_uint(a3);
        }
      }
      const bool tail = kb + 128 > p.Nkv;
      const bool diag = p.causal && (kb + 127 > r0[t] + off);
      if (tail || diag) {
        int lim = p.Nkv - 1 - kb;
        if (p.causal) lim = min(lim, row + off - kb);
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i > lim) s[c][i] = 0xFF800000u;
      }
      if (j + 1 < n[t]) {
        stage_ks(j + 1);
        if (j + 2 < n[t]) load_ks(j + 2);
      }
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        mx0 = fmax3(mx0, __uint_as_float(s[0][i]), __uint_as_float(s[0][i + 1]));
        mx1 = fmax3(mx1, __uint_as_float(s[1][i]), __uint_as_float(s[1][i + 1]));
        mx2 = fmax3(mx2, __uint_as_float(s[2][i]), __uint_as_float(s[2][i + 1]));
        mx3 = fmax3(mx3, __uint_as_float(s[3][i]), __uint_as_float(s[3][i + 1]));
      }
      // s_Q > 0, so max(y) * s_Q is the row max of x
      const float m_blk = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * qs_row;
      const bool grow = m_blk > m_ref + C::TAU;  // -inf + TAU = -inf: the first finite block moves it
      const bool had = m_ref != -INFINITY;
      float factor = 1.f;
      if (grow) {
        factor = had ? ex2(m_ref - m_blk) : 0.f;
        m_ref = m_blk;
      }
      const float negm = (m_ref == -INFINITY) ? 0.f : -m_ref;
      const uint64_t qs2 = f2(qs_row, qs_row), nm2 = f2(negm, negm);
      // P~ = e4m3(2^(x - m))
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          float a0, a1, a2, a3;
          f2_split(ffma2(f2(__uint_as_float(s[c][i]), __uint_as_float(s[c][i + 1])), qs2, nm2), a0, a1);
          f2_split(ffma2(f2(__uint_as_float(s[c][i + 2]), __uint_as_float(s[c][i + 3])), qs2, nm2), a2, a3);
          const uint32_t lo = e4m3x2_pair(ex2(a0), ex2(a1));
          const uint32_t hi = e4m3x2_pair(ex2(a2), ex2(a3));
          pk[c * 8 + i / 4] = lo | (hi << 16);
        }
      }
      if (j > 0) {
        // P V_t(j-1) and its row sum have read the P~ buffer and finished
        ok = wait_bar(smem_u32(&bars->pv_done[t]), (j - 1) & 1, abort_flag, p.timeout_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
      }
      tmem_st32(tbase + lane_off + C::T_P8 + 32 * t, pk);
      if (j > 0 && __any_sync(0xffffffffu, grow && had)) {
        // rescale O_t and l_t (blocks < j) to the new reference
        const float f = (grow && had) ? factor : 1.f;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
          tmem_st32(tO + cc * 32, o);
        }
        uint32_t lv = tmem_ld1(tL);
        tmem_ld_wait1(lv);
        tmem_st1(tL, __float_as_uint(__uint_as_float(lv) * f));
      }
      tmem_st_wait();
      __syncwarp();  // the staged key constants of block j + 1 are visible to the warp
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->p_full[t][j & 1]));
    }
    // ---------------------------------------------------------- epilogue
    if (ok && n[t] > 0) {
      ok = wait_bar(smem_u32(&bars->o_full[t]), 0, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) tc_fence_after();
    }
    if (ok) {
      float l = 0.f;  // no block visible: no row-sum MMA ran, the column is stale
      if (n[t] > 0) {
        uint32_t lv = tmem_ld1(tL);
        tmem_ld_wait1(lv);
        l = __uint_as_float(lv);
      }
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      const float* vs = p.v_scale + (size_t)bh * 128;
      float* orow = p.o + ((size_t)bh * p.Nq + row) * 128;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        if (n[t] > 0) {
          tmem_ld32(tO + cc * 32, o);
          tmem_ld_wait(o);
        }
        if (row < p.Nq) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 sv = *reinterpret_cast<const float4*>(vs + cc * 32 + i);
            float4 v;
            v.x = (l > 0.f) ? __uint_as_float(o[i + 0]) * sv.x * inv : 0.f;
            v.y = (l > 0.f) ? __uint_as_float(o[i + 1]) * sv.y * inv : 0.f;
            v.z = (l > 0.f) ? __uint_as_float(o[i + 2]) * sv.z * inv : 0.f;
            v.w = (l > 0.f) ? __uint_as_float(o[i + 3]) * sv.w * inv : 0.f;
            *reinterpret_cast<float4*>(orow + cc * 32 + i) = v;
          }
        }
      }
      if (row < p.Nq)
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
