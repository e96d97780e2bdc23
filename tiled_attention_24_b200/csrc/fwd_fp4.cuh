// FP4 (NVFP4) tiled attention forward for sm_100a: tcgen05 kind::mxf4nvf4
// block-scaled MMAs (e2m1 operands, one unsigned-e4m3 scale per 16 elements).
//
// "Hardware-Aware FP4 FlashAttention-4" page: the FP4 tensor cores multiply
// fast, but turning scores into FP4 probabilities -- exponentiate, find a
// block scale, divide, round -- stalls the pipeline; Direct-P maps the raw
// scores straight to the hardware codes instead.  Both P encodings are here:
//   p_mode 0, Direct-P:           P~ = e2m1_rne(6 * 2^(x - m)), block scale 1
//   p_mode 1, quantise-after-exp: p = 2^(x - m); per 16 keys
//                                 sf = e4m3_rne(amax(p) / 6), P~ = e2m1_rne(p / sf) * sf
// Steps per 128-key block j (tiling, masking and online softmax as in the
// bf16 kernel; the running max moves on every increase, so P <= 1):
//   S  = deq(Q) deq(K_j)^T               fp32 in TMEM (block-scaled MMA)
//   x  = S * scale * log2(e), masked
//   m, O and l rescaled by 2^(m_old - m) when the max grows
//   O += P~ deq(V_j)                     fp32 in TMEM (block-scaled MMA)
//   l += sum(P~)
//   O / l (fp32 output), LSE = ln2 * (m + log2(l / p_unit)), p_unit = 6 for
//   Direct-P (whose P~ approximates 6 * 2^(x - m)), 1 otherwise
//
// CTA = one (batch, head) x two 128-row query tiles; warps: 0 TMA producer,
// 1 MMA issuer, 2-3 idle (their registers go to the softmax warps through
// setmaxnreg), 4-7 softmax / correction / epilogue of tile 0, 8-11 of tile 1
// (thread = row).  The two tiles run concurrently, so each SM sub-partition
// has two softmax warps at independent phases: while one waits for an MMA or
// a barrier, or runs integer / fp32 work, the other keeps the exp pipe busy.
// Operands in shared memory (64-byte swizzled, K-major, 64 bytes = 128 e2m1
// codes per row): the two Q tiles, a ring of K and V^T tiles; each with its
// 1 KB of scale factors, which tcgen05.cp copies into TMEM in the layout the
// MMA reads (32 lanes x 16 bytes, replicated over the 4 lane quarters).  P is
// written by the softmax threads into a shared-memory tile per query tile
// (the A operand of a block-scaled MMA comes from shared memory),
// double-buffered, with its scale factors.
// TMEM: one score buffer S [0,128) shared by the tiles (its scores are moved
// to registers at once, then it is released to the other tile), O_0
// [128,256), O_1 [256,384), scale factors from column 384.  The next block's
// S of a tile is issued before that tile's current P V, so a softmax warp
// finds its next scores ready when it finishes a block.  The row sums l of
// the P values are accumulated by the tensor core too: P times a 16-column
// matrix of ones (e2m1 1.0, scale 1.0) into 16 TMEM columns per tile, so the
// softmax threads never decode their own codes.  d = 128 only.
#pragma once
#include "ptx.cuh"
#include "fwd_bf16.cuh"
#include "quant.cuh"

namespace ta {

struct FwdF4Params {
  const uint8_t* q_sf;  // [BH][ceil(Nq/128)][1 KB]
  const uint8_t* k_sf;  // [BH][KT][1 KB]
  const uint8_t* v_sf;  // [BH][KT][1 KB]
  float* o;             // [BH][Nq][128]
  float* lse;           // [BH][Nq]
  float* s_out;         // optional [BH][Nq][Nkv] scores (check of the block-scaled GEMM)
  int Nq, Nkv, n_qp, Tc, RTq, KT;  // n_qp: pairs of 128-row query tiles
  int causal, p_mode;
  float sl2;
  unsigned long long timeout_ns;
};

// kind::mxf4nvf4 instruction descriptor: A = B = e2m1 (1), K-major, scale
// factors ue4m3 (0), K = 64 per MMA.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

struct FwdF4Cfg {
  static constexpr int TILE = 128 * 64;  // 128 rows x 64 bytes of codes
  static constexpr int SF = 1024;
  static constexpr int SLOTB = 10240;    // codes + scales, 1 KB aligned
  static constexpr int NSLOT = 8;
  static constexpr int Q_OFF = 0;                      // Q_0, Q_1
  static constexpr int QSF_OFF = 2 * TILE;             // their scales
  static constexpr int SLOT_OFF = QSF_OFF + 2 * SF;    // 18 KB
  static constexpr int P_OFF = SLOT_OFF + NSLOT * SLOTB;  // [tile][buffer] P tiles
  static constexpr int PSF_OFF = P_OFF + 4 * TILE;        // [tile][buffer] P scales
  static constexpr int ONES_OFF = PSF_OFF + 4 * SF;      // 16 x 128 e2m1 ones (0x22 bytes)
  static constexpr int SF1_OFF = ONES_OFF + 1024;        // 512 bytes of scale 1.0 (0x38)
  static constexpr int RCP_OFF = SF1_OFF + 512;          // 128 floats: 1 / value of each e4m3 code
  static constexpr int BAR_OFF = RCP_OFF + 512;
  static constexpr int SMEM = BAR_OFF + 512 + 1024;
  static constexpr int THREADS = 384;
  // register split (launch: 384 threads x 168): warpgroup 0 drops to 72, the
  // two softmax warpgroups rise to 216: 128*72 + 256*216 = 64512 = 384*168
  static constexpr int REG_LOW = 72, REG_HIGH = 216;
  static constexpr uint32_t ID = idesc_nvf4(128, 128);
  static constexpr uint32_t ID_L = idesc_nvf4(128, 16);  // P x ones: row sums
  // TMEM columns: S, O_t, and the scale factors (8 columns = 2 MMA steps x 4)
  static constexpr uint32_t T_S = 0, T_O = 128;
  static constexpr uint32_t T_SFQ = 384;  // + 8 t
  static constexpr uint32_t T_SFK = 400;  // + 8 (j % 2)
  static constexpr uint32_t T_SFV = 416;  // + 8 (j % 2)
  static constexpr uint32_t T_SFP = 432;  // + 16 t + 8 (j % 2)
  static constexpr uint32_t T_SF1 = 464;  // scales of the ones matrix
  static constexpr uint32_t T_L = 480;    // + 16 t: row sums of tile t (column 0 is read)
};

struct FwdF4Bars {
  uint64_t q_full;
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint64_t s_full[2];     // MMA -> softmax of tile t: S_t(j) in the score buffer
  uint64_t s_free;        // softmax -> MMA: the score buffer's scores are in registers
  uint64_t p_full[2][2];  // [tile][j % 2]: P_t(j) and its scales in smem, O_t corrected
  uint64_t pv_done[2];    // [tile]: P V_t(j) finished
  uint64_t o_full[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(FwdF4Bars) <= 512, "barrier block too large");

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  if (!debug_check((dst & 15u) == 0 && (bytes & 15u) == 0 && (reinterpret_cast<uintptr_t>(src) & 15u) == 0)) return;
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// shared-memory descriptor with an explicit layout (0: no swizzle, 4: 64-byte swizzle)
__device__ __forceinline__ uint64_t smem_desc_l(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)layout << 61;
  return d;
}
// 32 rows x 16 bytes of shared memory -> TMEM, replicated to all 4 lane quarters
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
  if (!debug_check((taddr >> 16) == 0 && (taddr & 0xFFFFu) + 4u <= 512u)) return;
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
      : "memory");
}
// two non-negative fp32 -> e2m1 codes (one byte, `lo` in the low nibble)
__device__ __forceinline__ uint32_t e2m1x2_pos(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}
// two e2m1 codes (one byte) -> f16x2 values
__device__ __forceinline__ uint32_t e2m1x2_f16x2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(r) : "r"(byte));
  return r;
}
__device__ __forceinline__ uint32_t hadd2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ float f16x2_sum(uint32_t v) {
  float lo, hi;
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(v));
  return lo + hi;
}

template <bool SCORES_ONLY>
__global__ void __launch_bounds__(384, 1)
    fwd_fp4_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdF4Params p) {
  using C = FwdF4Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FwdF4Bars* bars = reinterpret_cast<FwdF4Bars*>(smem + C::BAR_OFF);
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
  // constant operands of the row-sum MMA: e2m1 ones (code 2) and their scales (1.0)
  for (int i = threadIdx.x; i < (1024 + 512) / 4; i += C::THREADS)
    *reinterpret_cast<uint32_t*>(smem + C::ONES_OFF + i * 4) = (i < 256) ? 0x22222222u : 0x38383838u;
  // reciprocals of the e4m3 block scales of P (quantise-after-exp), correctly
  // rounded once here instead of once per 16 keys in the softmax (0 for code 0)
  if (threadIdx.x < 128) {
    const float v = e4m3_value(threadIdx.x);
    reinterpret_cast<float*>(smem + C::RCP_OFF)[threadIdx.x] = (v > 0.f) ? __frcp_rn(v) : 0.f;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;
  auto kidx = [&](int j) { return SCORES_ONLY ? j : 2 * j; };
  auto vidx = [&](int j) { return 2 * j + 1; };

  if (warp < 4) {
   reg_dealloc<C::REG_LOW>();
   if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      if (!SCORES_ONLY) prefetch_tmap(&tmV);
      const uint32_t qbar = smem_u32(&bars->q_full);
      mbar_arrive_expect_tx(qbar, (present[1] ? 2 : 1) * (C::TILE + C::SF));
      for (int t = 0; t < 2; ++t) {
        if (!present[t]) continue;
        tma_load_3d(sbase + C::Q_OFF + t * C::TILE, &tmQ, qbar, 0, r0[t], bh);
        bulk_load(sbase + C::QSF_OFF + t * C::SF, p.q_sf + ((size_t)bh * p.RTq + 2 * qp + t) * C::SF, C::SF, qbar);
      }
      int it = 0;
      bool ok = true;
      for (int j = 0; j < nmax && ok; ++j) {
        for (int w = 0; w < (SCORES_ONLY ? 1 : 2) && ok; ++w, ++it) {
          const int slot = it % C::NSLOT;
          ok = wait_bar(smem_u32(&bars->kv_empty[slot]), ((it / C::NSLOT) & 1) ^ 1, abort_flag, p.timeout_ns);
          if (!ok) break;
          const uint32_t fb = smem_u32(&bars->kv_full[slot]);
          const uint32_t dst = sbase + C::SLOT_OFF + slot * C::SLOTB;
          mbar_arrive_expect_tx(fb, C::TILE + C::SF);
          if (w == 0) {
            tma_load_3d(dst, &tmK, fb, 0, j * 128, bh);
            bulk_load(dst + C::TILE, p.k_sf + ((size_t)bh * p.KT + j) * C::SF, C::SF, fb);
          } else {
            tma_load_3d(dst, &tmV, fb, j * 64, 0, bh);
            bulk_load(dst + C::TILE, p.v_sf + ((size_t)bh * p.KT + j) * C::SF, C::SF, fb);
          }
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
    // S sequence S_0(0), S_1(0), S_0(1), S_1(1), ... through the one score
    // buffer (each waits until the previous one's scores are in registers);
    // program order: prologue S_0(0), S_1(0), S_0(1); then per block j:
    // P V_0(j), S_1(j+1), P V_1(j), S_0(j+2).
    if (lane == 0) {
      bool ok = wait_bar(smem_u32(&bars->q_full), 0, abort_flag, p.timeout_ns);
      tc_fence_after();
      const uint64_t dQ0 = smem_desc_l(sbase + C::Q_OFF, 16, 512, 4);
      const uint64_t dSlot0 = smem_desc_l(sbase + C::SLOT_OFF, 16, 512, 4);
      const uint64_t dSf0 = smem_desc_l(sbase + C::SLOT_OFF + C::TILE, 16, 128, 0);
      const uint64_t dP0 = smem_desc_l(sbase + C::P_OFF, 16, 512, 4);
      const uint64_t dPsf0 = smem_desc_l(sbase + C::PSF_OFF, 16, 128, 0);
      const uint64_t dOnes = smem_desc_l(sbase + C::ONES_OFF, 16, 512, 4);
      if (ok) {
        const uint64_t dSf1 = smem_desc_l(sbase + C::SF1_OFF, 16, 128, 0);
        tc_cp_sf(tbase + C::T_SF1, dSf1);
        tc_cp_sf(tbase + C::T_SF1 + 4, dSf1);
        for (int t = 0; t < 2; ++t) {
          if (!present[t]) continue;
          const uint64_t dQsf = smem_desc_l(sbase + C::QSF_OFF + t * C::SF, 16, 128, 0);
          tc_cp_sf(tbase + C::T_SFQ + 8 * t, dQsf);
          tc_cp_sf(tbase + C::T_SFQ + 8 * t + 4, dQsf + (512 >> 4));
        }
      }
      int n_s = 0;  // S MMAs issued so far (the score buffer's uses)
      auto issue_S = [&](int t, int j) -> bool {
        if (n_s > 0) {
          if (!wait_bar(smem_u32(&bars->s_free), (n_s - 1) & 1, abort_flag, p.timeout_ns)) return false;
          tc_fence_after();
        }
        const int it = kidx(j), s = it % C::NSLOT;
        const uint64_t so = (uint64_t)(s * (C::SLOTB >> 4));
        const uint32_t sfk = tbase + C::T_SFK + (j & 1) * 8;
        const bool first = (t == 0) || (j >= n[0]);   // first user of K_j
        const bool last = (t == 1) || (j >= n[1]);    // last user of K_j
        if (first) {
          if (!wait_bar(smem_u32(&bars->kv_full[s]), (it / C::NSLOT) & 1, abort_flag, p.timeout_ns)) return false;
          tc_fence_after();
          tc_cp_sf(sfk, dSf0 + so);
          tc_cp_sf(sfk + 4, dSf0 + so + (512 >> 4));
        }
        const uint64_t dq = dQ0 + (uint64_t)(t * (C::TILE >> 4));
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)  // K = 64 e2m1 (32 bytes) per MMA
          mma_nvf4(tbase + C::T_S, dq + (uint64_t)(ks * 2), dSlot0 + so + (uint64_t)(ks * 2), C::ID,
                   tbase + C::T_SFQ + 8 * t + ks * 4, sfk + ks * 4, ks > 0);
        tc_commit(smem_u32(&bars->s_full[t]));
        if (last) tc_commit(smem_u32(&bars->kv_empty[s]));
        ++n_s;
        return true;
      };
      auto issue_PV = [&](int t, int j) -> bool {
        const int it = vidx(j), s = it % C::NSLOT;
        const uint64_t so = (uint64_t)(s * (C::SLOTB >> 4));
        const uint32_t sfv = tbase + C::T_SFV + (j & 1) * 8;
        const bool first = (t == 0) || (j >= n[0]);
        const bool last = (t == 1) || (j >= n[1]);
        if (first) {
          if (!wait_bar(smem_u32(&bars->kv_full[s]), (it / C::NSLOT) & 1, abort_flag, p.timeout_ns)) return false;
          tc_fence_after();
          tc_cp_sf(sfv, dSf0 + so);
          tc_cp_sf(sfv + 4, dSf0 + so + (512 >> 4));
        }
        if (!wait_bar(smem_u32(&bars->p_full[t][j & 1]), (j >> 1) & 1, abort_flag, p.timeout_ns)) return false;
        tc_fence_after();
        const int pb = t * 2 + (j & 1);
        const uint32_t sfp = tbase + C::T_SFP + pb * 8;
        const uint64_t pso = (uint64_t)(pb * (C::SF >> 4));
        tc_cp_sf(sfp, dPsf0 + pso);
        tc_cp_sf(sfp + 4, dPsf0 + pso + (512 >> 4));
        const uint64_t po = (uint64_t)(pb * (C::TILE >> 4));
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
          mma_nvf4(tbase + C::T_O + 128 * t, dP0 + po + (uint64_t)(ks * 2), dSlot0 + so + (uint64_t)(ks * 2), C::ID,
                   sfp + ks * 4, sfv + ks * 4, (j > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)  // l_t += P~ 1
          mma_nvf4(tbase + C::T_L + 16 * t, dP0 + po + (uint64_t)(ks * 2), dOnes + (uint64_t)(ks * 2), C::ID_L,
                   sfp + ks * 4, tbase + C::T_SF1 + ks * 4, (j > 0 || ks > 0) ? 1u : 0u);
        tc_commit(smem_u32(&bars->pv_done[t]));
        if (last) tc_commit(smem_u32(&bars->kv_empty[s]));
        if (j == n[t] - 1) tc_commit(smem_u32(&bars->o_full[t]));
        return true;
      };
      if (ok) {
        for (int t = 0; t < 2; ++t)
          if (!SCORES_ONLY && present[t] && n[t] == 0) tc_commit(smem_u32(&bars->o_full[t]));
      }
      if (ok && n[0] > 0) ok = issue_S(0, 0);
      if (ok && n[1] > 0) ok = issue_S(1, 0);
      if (ok && n[0] > 1) ok = issue_S(0, 1);
      for (int j = 0; j < nmax && ok; ++j) {
        if (!SCORES_ONLY && j < n[0] && !(ok = issue_PV(0, j))) break;
        if (j + 1 < n[1] && !(ok = issue_S(1, j + 1))) break;
        if (!SCORES_ONLY && j < n[1] && !(ok = issue_PV(1, j))) break;
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
    const float sl2 = p.sl2;
    const bool direct = p.p_mode == 0;
    const float* rcp_tab = reinterpret_cast<const float*>(smem + C::RCP_OFF);
    float m_ref = -INFINITY;  // l lives in TMEM (column tL), summed by the tensor core
    bool ok = present[t];
    if (!SCORES_ONLY && direct) {
      // Direct-P: every P block scale is 1.0 (0x38); this tile's two buffers, written once
      for (int i = threadIdx.x & 127; i < 2 * C::SF / 4; i += 128)
        *reinterpret_cast<uint32_t*>(smem + C::PSF_OFF + t * 2 * C::SF + i * 4) = 0x38383838u;
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
      if (SCORES_ONLY) {
        if (row < p.Nq) {
          float* dst = p.s_out + ((size_t)bh * p.Nq + row) * p.Nkv + kb;
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (kb + c * 32 + i < p.Nkv) dst[c * 32 + i] = __uint_as_float(s[c][i]);
        }
        continue;
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
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        mx0 = fmax3(mx0, __uint_as_float(s[0][i]), __uint_as_float(s[0][i + 1]));
        mx1 = fmax3(mx1, __uint_as_float(s[1][i]), __uint_as_float(s[1][i + 1]));
        mx2 = fmax3(mx2, __uint_as_float(s[2][i]), __uint_as_float(s[2][i + 1]));
        mx3 = fmax3(mx3, __uint_as_float(s[3][i]), __uint_as_float(s[3][i + 1]));
      }
      const float m_blk = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
      const bool grow = m_blk > m_ref;  // the reference moves on every increase
      const bool had = m_ref != -INFINITY;
      float factor = 1.f;
      if (grow) {
        factor = had ? ex2(m_ref - m_blk) : 0.f;
        m_ref = m_blk;
      }
      const float negm = (m_ref == -INFINITY) ? 0.f : -m_ref;
      // ---- P codes (row rr of the P tile, 64 bytes, 64-byte swizzle) and scales.
      // Buffer j % 2 was last read by P V_t(j-2), which finished before S_t(j)
      // was computed (the S_t(j) commit covers every earlier MMA).
      uint8_t* ptile = smem + C::P_OFF + (t * 2 + (j & 1)) * C::TILE + rr * 64;
      uint8_t* psf = smem + C::PSF_OFF + (t * 2 + (j & 1)) * C::SF;
      // Direct-P: 6 * 2^(x - m) = 2^(x - m + log2 6), one exponential per score
      const float neg_arg = direct ? negm + 2.5849625007211562f : negm;
      // p = 2^(x - m) (times 6 for Direct-P) for the whole row, in place
      const uint64_t sl2x2 = f2(sl2, sl2), na2 = f2(neg_arg, neg_arg);
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float a0, a1;
          f2_split(ffma2(f2(__uint_as_float(s[c][i]), __uint_as_float(s[c][i + 1])), sl2x2, na2), a0, a1);
          s[c][i] = __float_as_uint(ex2(a0));
          s[c][i + 1] = __float_as_uint(ex2(a1));
        }
      // quantise-after-exp: the 8 block scales of the row first (independent
      // chains), then codes of p * (1 / sf): within an ulp of p / sf, so only a
      // value on an e2m1 rounding boundary can round differently; a zero scale
      // (an all-zero block) gives zero codes
      float rs[8];
      if (!direct) {
#pragma unroll
        for (int blk = 0; blk < 8; ++blk) {
          const uint32_t* v = &s[blk >> 1][(blk & 1) * 16];
          const float a0 = fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
          const float a1 = fmax3(__uint_as_float(v[3]), __uint_as_float(v[4]), __uint_as_float(v[5]));
          const float a2 = fmax3(__uint_as_float(v[6]), __uint_as_float(v[7]), __uint_as_float(v[8]));
          const float a3 = fmax3(__uint_as_float(v[9]), __uint_as_float(v[10]), __uint_as_float(v[11]));
          const float a4 = fmax3(__uint_as_float(v[12]), __uint_as_float(v[13]), __uint_as_float(v[14]));
          const float amax = fmax3(fmax3(a0, a1, a2), fmax3(a3, a4, __uint_as_float(v[15])), 0.f);
          const uint32_t sfc = (amax > 0.f) ? e4m3_rne(__fdiv_rn(fmaxf(amax, 1e-30f), 6.f)) : 0u;
          psf[sf_offset(rr, blk)] = (uint8_t)sfc;
          rs[blk] = rcp_tab[sfc];  // p <= 1, so amax / 6 <= 1/6 and sfc < 128
        }
      }
#pragma unroll
      for (int blk = 0; blk < 8; ++blk) {  // 16 keys per block
        const int c = blk >> 1, i0 = (blk & 1) * 16;
        float v[16];
        if (direct) {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(s[c][i0 + e]);
        } else {
          const uint64_t r2 = f2(rs[blk], rs[blk]);
#pragma unroll
          for (int e = 0; e < 16; e += 2)
            f2_split(fmul2(f2(__uint_as_float(s[c][i0 + e]), __uint_as_float(s[c][i0 + e + 1])), r2), v[e], v[e + 1]);
        }
        uint32_t b[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) b[e] = e2m1x2_pos(v[2 * e], v[2 * e + 1]);
        const uint32_t w0 = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
        const uint32_t w1 = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
        // 8 bytes = keys [16 blk, 16 blk + 16) -> chunk blk / 2, half blk % 2
        const int chunk = blk >> 1;
        uint8_t* dst = ptile + ((chunk ^ ((rr >> 1) & 3)) << 4) + (blk & 1) * 8;
        *reinterpret_cast<uint2*>(dst) = make_uint2(w0, w1);
      }
      if (j > 0 && __any_sync(0xffffffffu, grow && had)) {
        // rescale O_t and l_t (blocks < j) to the new reference
        ok = wait_bar(smem_u32(&bars->pv_done[t]), (j - 1) & 1, abort_flag, p.timeout_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
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
        tmem_st_wait();
      }
      fence_proxy_async_smem();  // P tile and scales are read by the tensor core
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->p_full[t][j & 1]));
    }
    // ---------------------------------------------------------- epilogue
    if (!SCORES_ONLY && ok) {
      ok = wait_bar(smem_u32(&bars->o_full[t]), 0, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        float l = 0.f;  // no block visible: no row-sum MMA ran, the column is stale
        if (n[t] > 0) {
          uint32_t lv = tmem_ld1(tL);
          tmem_ld_wait1(lv);
          l = __uint_as_float(lv);
        }
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        float* orow = p.o + ((size_t)bh * p.Nq + row) * 128;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_ld_wait(o);
          if (row < p.Nq) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              float4 v;
              v.x = (l > 0.f) ? __uint_as_float(o[i + 0]) * inv : 0.f;
              v.y = (l > 0.f) ? __uint_as_float(o[i + 1]) * inv : 0.f;
              v.z = (l > 0.f) ? __uint_as_float(o[i + 2]) * inv : 0.f;
              v.w = (l > 0.f) ? __uint_as_float(o[i + 3]) * inv : 0.f;
              *reinterpret_cast<float4*>(orow + cc * 32 + i) = v;
            }
          }
        }
        if (row < p.Nq)
          // Direct-P values are 6 * 2^(x - m): LSE = m + log2(l / 6)
          p.lse[(size_t)bh * p.Nq + row] =
              (l > 0.f) ? (m_ref + log2f(l) - (direct ? 2.5849625007211562f : 0.f)) * 0.69314718055994531f
                        : -INFINITY;
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
