// bf16 tiled attention forward for sm_100a (TMA + tcgen05 + TMEM).
//
// What it computes ("Can a full-day context beat one minute? Flash attention
// and the sequence-length question", sections "The Flash Attention algorithm"
// and "Online softmax recurrence"): O = softmax(scale * Q K^T) V and the
// natural-log LSE per query row, with Q split into B_r = 128-row blocks and
// K/V into B_c = 128-key blocks; S_ij = Q_i K_j^T lives only in tensor memory,
// the running row max m, running sum l and the unnormalised O accumulator are
// updated block by block and O is divided by l once at the end ("FA2" item 1).
//
// CTA = one (batch, head) and TWO query tiles of 128 rows (256 rows).  Roles
// (warp specialisation, "FlashAttention 4" section "What is new"):
//   warp 0      TMA producer: Q tiles once, then K_j, V_j into a smem ring
//               (Q and K_0 issued before the CTA-wide barrier; near its end
//               it prefetches into L2 the first tiles of the CTA one wave
//               later, the likely next occupant of the SM)
//   warp 1      MMA issuer (one thread): S_t = Q_t K_j^T and O_t += P_t V_j
//   warps 2-3   idle (they complete warpgroup 0, whose registers are handed
//               to the softmax warpgroups with setmaxnreg)
//   warps 4-7   softmax warpgroup of query tile 0 (thread = TMEM lane = row)
//   warps 8-11  softmax warpgroup of query tile 1
// The two softmax warpgroups ping-pong: while one turns S into P, the tensor
// core runs the other tile's P V and next S ("FA3" item 2, interleaving matmul
// and softmax).  Each softmax warpgroup also does its own (rare, lazy) O
// correction and the epilogue (O / l -> bf16 -> smem -> TMA store, LSE).
//
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   S_t  : columns [128 t, 128 t + 128)   fp32 scores of tile t
//   P_t  : columns [128 t, 128 t + 64)    bf16x2 probabilities, aliasing S_t
//   O_t  : columns [256 + D t, 256 + D t + D)   fp32 accumulator of tile t
//
// Variable-length batches (VARLEN = true; "FlashAttention 4" page, what is
// missing: varlen): sequences packed token-major, Q/O [total_q][H][D],
// K/V [total_k][H_kv][D], sequence b holding rows [cu_q[b], cu_q[b+1]) and
// keys [cu_k[b], cu_k[b+1]); LSE [H][total_q].  The TMA maps view the packed
// tensors as (D, heads, tokens) with boxes of 64 x 1 x 128, which land in
// shared memory exactly like the dense (D, N, B*H) boxes of 64 x 128 x 1.
// Rows of a tile past the sequence's end belong to the next sequence (or read
// as zero past the tensor): their keys are masked like a ragged tail, their
// query rows are not stored (the epilogue writes rows directly instead of a
// TMA store, which would overwrite the next sequence).
//
// Shared memory (128-byte swizzled, the TMA and UMMA canonical layout): each
// 128 x D bf16 tile is stored as D/64 column blocks of 128 rows x 128 bytes.
// Q0, Q1, then a ring of NSTAGE stages; stage i holds V_{i-1} (first tile)
// and K_i (second tile), the two operands a KV step consumes together, so
// the MMA thread waits on one barrier per step.
#pragma once
#include "ptx.cuh"

// Speculative barrier tests inside MMA groups (hide a wait's latency behind
// the group's last MMA).  Off: every mbarrier operation of the issuing thread
// first waits for its queued MMAs to drain, so the test itself leaves a
// bubble in the tensor pipe (measured: ~70 cycles per group).
#ifndef TA_SPEC_TEST
#define TA_SPEC_TEST 0
#endif
#ifndef TA_POLY_PERIOD
#define TA_POLY_PERIOD 4
#endif
#ifndef TA_POLY_PAIRS
#define TA_POLY_PAIRS 0
#endif
// P handed to the P V MMA in TA_P_SPLIT parts (1, 2 or 4) at d = 128
#ifndef TA_P_SPLIT
#define TA_P_SPLIT 2
#endif
#define TA_P_HALVES (TA_P_SPLIT > 1)
#ifndef TA_POLY_PAIRS_D64
#define TA_POLY_PAIRS_D64 TA_POLY_PAIRS
#endif

namespace ta {

struct FwdParams {
  float* lse;
  int Nq, Nkv, n_qp, Tc;
  int group;  // query heads per key/value head (grouped-query attention; 1 = plain)
  int causal;
  float sl2;  // scale * log2(e)
  unsigned long long timeout_ns;
  // variable-length batches only
  const int* cu_q;  // [nb + 1] row offsets of the sequences in the packed Q / O
  const int* cu_k;  // [nb + 1] key offsets in the packed K / V
  uint16_t* o;      // packed O [total_q][H][D]
  int nb, H, total_q, total_k;
  int wave;  // CTAs resident at once (one per SM): CTA b prefetches CTA b + wave's first tiles into L2
};

template <int D>
struct FwdCfg {
  static constexpr int BR = 128, BC = 128;
  static constexpr int TILE = 128 * D * 2;       // bytes of one 128 x D bf16 tile
  static constexpr int HALF = 128 * 128;         // one 64-column block (128 rows x 128 B)
  static constexpr int NSTAGE = (D == 128) ? 2 : 5;
  static constexpr int STAGE = 2 * TILE;
  static constexpr int Q_OFF = 0;
  static constexpr int SLOT_OFF = 2 * TILE;
  static constexpr int BAR_OFF = SLOT_OFF + NSTAGE * STAGE;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = BAR_OFF + BAR_BYTES + 1024;  // + alignment slack
  static constexpr int THREADS = 384;
  // register split (launch: 384 threads x 168): warpgroup 0 drops to 80 (72
  // at d = 64), the two softmax warpgroups rise to 208 (216):
  // 128*80 + 256*208 = 63488 and 128*72 + 256*216 = 64512 <= 384*168
  static constexpr int REG_LOW = (D == 64) ? 72 : 80, REG_HIGH = (D == 64) ? 216 : 208;
  // d = 64: P gets its own TMEM columns (S_0, S_1 [0,256), P_0, P_1 [256,384),
  // O_0, O_1 [384,512)), so a tile's next S is issued as soon as its softmax
  // holds the current scores, not after its P V.  d = 128: no room; P aliases S.
  static constexpr bool SEP_P = (D == 64);
  static constexpr uint32_t T_P = SEP_P ? 256 : 0, T_O = SEP_P ? 384 : 256;
  static constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, false);
  static constexpr uint32_t ID_PV = idesc_bf16_f32(128, D, true);
  static constexpr float TAU = 8.0f;  // lazy-rescale threshold, log2 units
  // of every POLY_PERIOD element pairs, POLY_PAIRS take 2^x from the cubic
  static constexpr int POLY_PERIOD = TA_POLY_PERIOD, POLY_PAIRS = (D == 64) ? TA_POLY_PAIRS_D64 : TA_POLY_PAIRS;
};

struct FwdBars {
  uint64_t q_full;
  uint64_t kv_full[5];
  uint64_t kv_empty[5];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t p_part[2][3];  // d = 128: P of the first k + 1 of TA_P_SPLIT key parts stored
  uint64_t o_full[2];
  uint64_t epi[2];
  uint64_t s_free[2];   // d = 64: scores of tile t are in registers
  uint64_t pv_done[2];  // d = 64: P V_t(j) finished (P_t columns free, O_t settled)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(FwdBars) <= 256, "barrier block too large");

__device__ __forceinline__ int fwd_tile_kv_count(int r0, int Nq, int Nkv, int Tc, int causal) {
  if (r0 >= Nq) return 0;
  if (!causal) return Tc;
  const long long r_last = min(r0 + 127, Nq - 1);
  const long long last_key = r_last + (long long)(Nkv - Nq);
  if (last_key < 0) return 0;
  return (int)min((long long)Tc, last_key / 128 + 1);
}

// Bounded wait that ignores the abort flag (used to drain work in flight).
__device__ __forceinline__ bool wait_bar_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  int dummy = 0;
  return wait_bar(bar, parity, &dummy, limit_ns);
}

template <int D, bool VARLEN = false>
__global__ void __launch_bounds__(384, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + C::BAR_OFF);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: (batch*head, pair of query tiles); heaviest pairs first when causal
  // non-causal: a head's query pairs are consecutive (its K/V stay in L2);
  // causal: all heads' heaviest pairs first (longest-processing-time order)
  const int BH = gridDim.x / p.n_qp;
  const int bh = p.causal ? (int)(blockIdx.x % BH) : (int)(blockIdx.x / p.n_qp);
  const int qp = p.causal ? p.n_qp - 1 - (int)(blockIdx.x / BH) : (int)(blockIdx.x % p.n_qp);
  int Nq = p.Nq, Nkv = p.Nkv, Tc = p.Tc;
  int qstart = 0, kstart = 0, head = bh;  // varlen: first row / key of the sequence, query head
  if constexpr (VARLEN) {
    const int b = bh / p.H;
    head = bh % p.H;
    // offsets clamped to the tensors, so that a bad offset array cannot
    // move a store out of the packed O
    qstart = min(max(p.cu_q[b], 0), p.total_q);
    Nq = min(max(p.cu_q[b + 1], qstart), p.total_q) - qstart;
    kstart = min(max(p.cu_k[b], 0), p.total_k);
    Nkv = min(max(p.cu_k[b + 1], kstart), p.total_k) - kstart;
    Tc = (Nkv + 127) / 128;
    if (qp * 256 >= Nq) return;  // the whole CTA: nothing initialised yet
  }
  int r0[2], n[2];
  bool present[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    r0[t] = qp * 256 + t * 128;
    present[t] = r0[t] < Nq;
    n[t] = fwd_tile_kv_count(r0[t], Nq, Nkv, Tc, p.causal);
  }
  const int nmax = max(n[0], n[1]);
  volatile int* abort_flag = &bars->abort;
  if (TA_DEBUG && threadIdx.x == 0 && p.causal)  // key tiles this CTA's query tiles never visit
    debug_count(TA_CNT_SKIPPED_TILES, (present[0] ? Tc - n[0] : 0) + (present[1] ? Tc - n[1] : 0));

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(smem_u32(&bars->kv_full[s]), 1);
      mbar_init(smem_u32(&bars->kv_empty[s]), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&bars->s_full[t]), 1);
      mbar_init(smem_u32(&bars->p_full[t]), 128);
      for (int k = 0; k < 3; ++k) mbar_init(smem_u32(&bars->p_part[t][k]), 128);
      mbar_init(smem_u32(&bars->o_full[t]), 1);
      mbar_init(smem_u32(&bars->epi[t]), 128);
      mbar_init(smem_u32(&bars->s_free[t]), 128);
      mbar_init(smem_u32(&bars->pv_done[t]), 1);
    }
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    fence_mbar_init();
    // the producer thread starts the Q and K_0 copies before the CTA-wide
    // barrier, so that their latency overlaps the TMEM allocation (the barrier
    // words it just wrote are made visible to the async proxy first)
    fence_proxy_async_smem();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    const uint32_t qbar = smem_u32(&bars->q_full);
    mbar_arrive_expect_tx(qbar, (present[0] + present[1]) * C::TILE);
    for (int t = 0; t < 2; ++t) {
      if (!present[t]) continue;
      for (int h = 0; h < D / 64; ++h) {
        if constexpr (VARLEN)
          tma_load_3d(sbase + C::Q_OFF + t * C::TILE + h * C::HALF, &tmQ, qbar, h * 64, head, qstart + r0[t]);
        else
          tma_load_3d(sbase + C::Q_OFF + t * C::TILE + h * C::HALF, &tmQ, qbar, h * 64, r0[t], bh);
      }
    }
    if (nmax > 0) {  // stage 0: K_0 only (its slot has never been used: no empty wait)
      const uint32_t fb = smem_u32(&bars->kv_full[0]);
      mbar_arrive_expect_tx(fb, C::TILE);
      const int kvh0 = head / p.group;
      for (int h = 0; h < D / 64; ++h) {
        if constexpr (VARLEN)
          tma_load_3d(sbase + C::SLOT_OFF + C::TILE + h * C::HALF, &tmK, fb, h * 64, kvh0, kstart);
        else
          tma_load_3d(sbase + C::SLOT_OFF + C::TILE + h * C::HALF, &tmK, fb, h * 64, 0, kvh0);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;

  if (warp < 4) {
   reg_dealloc<C::REG_LOW>();
   if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      const uint32_t qbar = smem_u32(&bars->q_full);
      const int kvh = head / p.group;  // key/value head of this query head
      // stage i (0..nmax): V_{i-1} at +0 (none for i = 0), K_i at +TILE (none
      // for i = nmax); stage 0 was issued before the CTA-wide barrier
      int it = 1, slot = 1 % C::NSTAGE;
      uint32_t ph = (C::NSTAGE == 1) ? 1u : 0u;
      bool ok = true;
      for (int i = 1; nmax > 0 && i <= nmax && ok; ++i, ++it, (++slot == C::NSTAGE) ? (slot = 0, ph ^= 1u) : 0u) {
        ok = wait_bar(smem_u32(&bars->kv_empty[slot]), ph ^ 1, abort_flag, p.timeout_ns);
        if (!ok) break;
        if (!VARLEN && p.wave > 0 && i == max(1, nmax - 4) && blockIdx.x + p.wave < gridDim.x) {
          // the CTA that will most likely take this SM next (one wave later):
          // its Q tiles and first K tile into L2 now
          const int nb2 = blockIdx.x + p.wave;
          const int bh2 = p.causal ? (int)(nb2 % BH) : (int)(nb2 / p.n_qp);
          const int qp2 = p.causal ? p.n_qp - 1 - (int)(nb2 / BH) : (int)(nb2 % p.n_qp);
          for (int t = 0; t < 2; ++t)
            if (qp2 * 256 + t * 128 < Nq)
              for (int h = 0; h < D / 64; ++h) tma_prefetch_3d(&tmQ, h * 64, qp2 * 256 + t * 128, bh2);
          for (int h = 0; h < D / 64; ++h) tma_prefetch_3d(&tmK, h * 64, 0, bh2 / p.group);
        }
        const uint32_t fb = smem_u32(&bars->kv_full[slot]);
        mbar_arrive_expect_tx(fb, ((i > 0) + (i < nmax)) * C::TILE);
        const uint32_t dst = sbase + C::SLOT_OFF + slot * C::STAGE;
        for (int h = 0; h < D / 64; ++h) {
          if constexpr (VARLEN) {
            if (i > 0) tma_load_3d(dst + h * C::HALF, &tmV, fb, h * 64, kvh, kstart + (i - 1) * 128);
            if (i < nmax) tma_load_3d(dst + C::TILE + h * C::HALF, &tmK, fb, h * 64, kvh, kstart + i * 128);
          } else {
            if (i > 0) tma_load_3d(dst + h * C::HALF, &tmV, fb, h * 64, (i - 1) * 128, kvh);
            if (i < nmax) tma_load_3d(dst + C::TILE + h * C::HALF, &tmK, fb, h * 64, i * 128, kvh);
          }
        }
      }
      // Never leave a copy in flight: wait for the last load of every stage.
      if (!ok) {
        wait_bar_drain(qbar, 0, p.timeout_ns);
        for (int back = 1; back <= C::NSTAGE && it - back >= 0; ++back) {
          const int i2 = it - back;
          wait_bar_drain(smem_u32(&bars->kv_full[i2 % C::NSTAGE]), (i2 / C::NSTAGE) & 1, p.timeout_ns);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    // The tensor pipe holds little beyond the MMA in flight, so anything the
    // issuing thread does between two MMAs idles it.  Hence: descriptors are
    // built once (one 64-bit add per MMA), slot/phase counters advance
    // incrementally, and the barrier of the NEXT group is tested (without
    // blocking) just before the last MMA of the current group is issued, so
    // that the test's latency hides behind that MMA.
    if (lane == 0) {
      bool ok = spin_bar(smem_u32(&bars->q_full), 0, abort_flag, p.timeout_ns);
      const uint64_t dQ0 = smem_desc(sbase + C::Q_OFF, 16, 1024);
      const uint64_t dQ1 = smem_desc(sbase + C::Q_OFF + C::TILE, 16, 1024);
      const uint64_t dV0 = smem_desc(sbase + C::SLOT_OFF, C::HALF, 1024);
      const uint64_t dK0 = smem_desc(sbase + C::SLOT_OFF + C::TILE, 16, 1024);
      // Issue one S group (K in stage st); before its last MMA, test barrier (nb, np).
      auto issue_S = [&](int t, int st, uint32_t nb, uint32_t np) -> bool {
        const uint64_t dq = t ? dQ1 : dQ0;
        const uint64_t dk = dK0 + (uint64_t)(st * (C::STAGE >> 4));
        const uint32_t dS = tbase + t * 128;
        bool ready = TA_SPEC_TEST != 0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * C::HALF + (kk & 3) * 32) >> 4);
          if (TA_SPEC_TEST && kk == D / 16 - 1 && nb) ready = mbar_test_wait(nb, np);
          mma_f16_ss(dS, dq + off, dk + off, C::ID_S, kk > 0);
        }
        tc_commit(smem_u32(&bars->s_full[t]));
        return ready;
      };
      auto issue_PV = [&](int t, int st, int j, uint32_t nb, uint32_t np) -> bool {
        const uint64_t dv = dV0 + (uint64_t)(st * (C::STAGE >> 4));
        const uint32_t dO = tbase + C::T_O + t * D, aP = tbase + (C::SEP_P ? C::T_P + 64 * t : 128 * t);
        const uint32_t acc0 = (j > 0) ? 1u : 0u;
        bool ready = TA_SPEC_TEST != 0;
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk) {
          if (TA_SPEC_TEST && kk == 7 && nb) ready = mbar_test_wait(nb, np);
          mma_f16_ts(dO, aP + kk * 8, dv + (uint64_t)(kk * (2048 >> 4)), C::ID_PV, kk > 0 ? 1u : acc0);
        }
        return ready;
      };
      // Barrier waits poll without suspending (spin_bar): a suspended
      // try_wait can resume a few hundred cycles after the phase completes,
      // and the softmax of the other tile is on the critical path behind it.
      // A barrier the softmax arrives at (after writing or reading tensor
      // memory) needs the tcgen05 fence; a TMA barrier does not (TMA writes
      // and MMA operand reads are both in the async proxy, ordered by the
      // barrier's transaction count).
      auto need = [&](bool seen, uint32_t bar, uint32_t par) -> bool {
        if (!seen && !spin_bar(bar, par, abort_flag, p.timeout_ns)) return false;
        tc_fence_after();
        return true;
      };
      auto need_tma = [&](bool seen, uint32_t bar, uint32_t par) -> bool {
        return seen || spin_bar(bar, par, abort_flag, p.timeout_ns);
      };
      // d = 128 with P in TA_P_SPLIT parts: the MMAs of part k once the
      // softmax has stored it, so the first parts run while it computes the rest
      auto issue_PV_halves = [&](int t, int st, int j) -> bool {
        const uint64_t dv = dV0 + (uint64_t)(st * (C::STAGE >> 4));
        const uint32_t dO = tbase + C::T_O + t * D, aP = tbase + 128 * t;
        const uint32_t acc0 = (j > 0) ? 1u : 0u;
        constexpr int PER = 8 / TA_P_SPLIT;
#pragma unroll
        for (int k = 0; k < TA_P_SPLIT; ++k) {
          const uint32_t bar = (k < TA_P_SPLIT - 1) ? smem_u32(&bars->p_part[t][k]) : smem_u32(&bars->p_full[t]);
          if (!need(false, bar, j & 1)) return false;
#pragma unroll
          for (int kk = k * PER; kk < (k + 1) * PER; ++kk)
            mma_f16_ts(dO, aP + kk * 8, dv + (uint64_t)(kk * (2048 >> 4)), C::ID_PV, kk > 0 ? 1u : acc0);
        }
        return true;
      };
      const uint32_t pf0 = smem_u32(&bars->p_full[0]), pf1 = smem_u32(&bars->p_full[1]);
      int st = 0;        // stage of the current step (slot), its phase
      uint32_t sp = 0;
      if (ok && nmax > 0) {
        ok = spin_bar(smem_u32(&bars->kv_full[0]), 0, abort_flag, p.timeout_ns);
        if (ok) {
          if (n[0] > 0) issue_S(0, 0, 0, 0);
          if (n[1] > 0) issue_S(1, 0, 0, 0);
          tc_commit(smem_u32(&bars->kv_empty[0]));
        }
      }
      if (ok) {
        for (int t = 0; t < 2; ++t)
          if (present[t] && n[t] == 0) tc_commit(smem_u32(&bars->o_full[t]));
      }
      // step j uses stage j + 1: V_j for both P V groups, K_{j+1} for the next S
      if constexpr (C::SEP_P) {
        const uint32_t sf0 = smem_u32(&bars->s_free[0]), sf1 = smem_u32(&bars->s_free[1]);
        bool seenSt = false;
        for (int j = 0; j < nmax && ok; ++j) {
          if (++st == C::NSTAGE) { st = 0; sp ^= 1u; }
          if (!(ok = need_tma(seenSt, smem_u32(&bars->kv_full[st]), sp))) break;
          int st1 = st + 1;
          uint32_t sp1 = sp;
          if (st1 == C::NSTAGE) { st1 = 0; sp1 ^= 1u; }
          const uint32_t nbar = (j + 1 < nmax) ? smem_u32(&bars->kv_full[st1]) : 0u;
          // each tile's next S as soon as its softmax holds the current scores
          if (j + 1 < n[0]) {
            if (!(ok = need(false, sf0, j & 1))) break;
            issue_S(0, st, 0, 0);
          }
          if (j + 1 < n[1]) {
            if (!(ok = need(false, sf1, j & 1))) break;
            issue_S(1, st, 0, 0);
          }
          if (j < n[0]) {
            if (!(ok = need(false, pf0, j & 1))) break;
            issue_PV(0, st, j, 0, 0);
            tc_commit(smem_u32(&bars->pv_done[0]));
            if (j == n[0] - 1) tc_commit(smem_u32(&bars->o_full[0]));
          }
          seenSt = false;
          if (j < n[1]) {
            if (!(ok = need(false, pf1, j & 1))) break;
            seenSt = issue_PV(1, st, j, nbar, sp1);
            tc_commit(smem_u32(&bars->pv_done[1]));
            if (j == n[1] - 1) tc_commit(smem_u32(&bars->o_full[1]));
          }
          seenSt = seenSt && nbar;
          tc_commit(smem_u32(&bars->kv_empty[st]));
        }
      } else {
        bool seenSt = false;
        for (int j = 0; j < nmax && ok; ++j) {
          if (++st == C::NSTAGE) { st = 0; sp ^= 1u; }
          if (!(ok = need_tma(seenSt, smem_u32(&bars->kv_full[st]), sp))) break;
          int st1 = st + 1;
          uint32_t sp1 = sp;
          if (st1 == C::NSTAGE) { st1 = 0; sp1 ^= 1u; }
          const uint32_t nbar = (j + 1 < nmax) ? smem_u32(&bars->kv_full[st1]) : 0u;
          bool seenP1 = false;
          if (j < n[0]) {
            if (TA_P_HALVES) {
              if (!(ok = issue_PV_halves(0, st, j))) break;
            } else {
              if (!(ok = need(false, pf0, j & 1))) break;
              seenP1 = issue_PV(0, st, j, (j < n[1]) ? pf1 : 0u, j & 1);
            }
            if (j == n[0] - 1) tc_commit(smem_u32(&bars->o_full[0]));
          }
          if (j + 1 < n[0]) seenP1 = issue_S(0, st, (!seenP1 && j < n[1]) ? pf1 : 0u, j & 1) || seenP1;
          seenSt = false;
          if (j < n[1]) {
            if (TA_P_HALVES) {
              if (!(ok = issue_PV_halves(1, st, j))) break;
            } else {
              if (!(ok = need(seenP1, pf1, j & 1))) break;
              seenSt = issue_PV(1, st, j, nbar, sp1);
            }
            if (j == n[1] - 1) tc_commit(smem_u32(&bars->o_full[1]));
          }
          if (j + 1 < n[1]) seenSt = issue_S(1, st, seenSt ? 0u : nbar, sp1) || seenSt;
          seenSt = seenSt && nbar;
          tc_commit(smem_u32(&bars->kv_empty[st]));
        }
      }
      if (!ok) {
        // drain: every MMA issued so far must finish before TMEM is freed
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
    const int rr = quarter * 32 + lane;  // row within the tile == TMEM lane
    const int row = r0[t] + rr;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tbase + lane_off + t * 128;
    const uint32_t tO = tbase + lane_off + C::T_O + t * D;
    const uint32_t tP = C::SEP_P ? tbase + lane_off + C::T_P + 64 * t : tS;
    const float sl2 = p.sl2;
    const int off = Nkv - Nq;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = present[t];
    for (int j = 0; j < n[t] && ok; ++j) {
      ok = wait_bar(smem_u32(&bars->s_full[t]), j & 1, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t s[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, s[c]);
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_wait(s[c]);
      if constexpr (C::SEP_P) {
        tc_fence_before();
        mbar_arrive(smem_u32(&bars->s_free[t]));  // the MMA may now compute S_t(j+1) here
      }
      const int kb = j * 128;
      const bool tail = kb + 128 > Nkv;
      const bool diag = p.causal && (kb + 127 > r0[t] + off);
      if (tail || diag) {
        int lim = Nkv - 1 - kb;                         // last visible column of this row
        if (p.causal) lim = min(lim, row + off - kb);
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i > lim) s[c][i] = 0xFF800000u;  // -inf
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
      // lazy rescale: move the reference max only when it rises by more than TAU
      const bool need = m_blk > m_ref + C::TAU;
      if (TA_DEBUG) {  // rows whose reference moved after their first key block
        const unsigned moved = __ballot_sync(__activemask(), need && m_ref != -INFINITY);
        if (lane == 0) debug_count(TA_CNT_RESCALES, __popc(moved));
      }
      float factor = 1.f;
      if (need) {
        factor = ex2(m_ref - m_blk);  // 0 when m_ref == -inf
        l *= factor;
        m_ref = m_blk;
      }
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        if constexpr (C::SEP_P) {
          // P V_t(j-1) must be done with O_t (with P aliasing S, the S_t(j)
          // commit already implied it)
          ok = wait_bar(smem_u32(&bars->pv_done[t]), (j - 1) & 1, abort_flag, p.timeout_ns);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
        }
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
          tmem_st32(tO + cc * 32, o);
        }
      }
      const float negm = (m_ref == -INFINITY) ? 0.f : -m_ref;
      const uint64_t sl2x2 = f2(sl2, sl2), negmx2 = f2(negm, negm);
      uint64_t lsA = f2(0.f, 0.f), lsB = f2(0.f, 0.f);
      uint32_t pk[2][32];
      if ((tail || diag) || C::POLY_PAIRS == 0) {
        // hardware ex2 throughout (masked tiles: -inf scores must give exactly 0)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0, x1;
            f2_split(ffma2(f2(__uint_as_float(s[c][2 * i]), __uint_as_float(s[c][2 * i + 1])), sl2x2, negmx2), x0,
                     x1);
            const float p0 = ex2(x0), p1 = ex2(x1);
            if (i & 1) lsB = fadd2(lsB, f2(p0, p1));
            else lsA = fadd2(lsA, f2(p0, p1));
            pk[c >> 1][(c & 1) * 16 + i] = pack_bf16(p0, p1);
          }
          if (TA_P_HALVES && !C::SEP_P && c < 3 && ((c + 1) % (4 / TA_P_SPLIT)) == 0) {
            // keys up to 32 (c + 1): the MMA thread may start P V on this part
            // now (its TMEM columns held scores already in registers)
            constexpr int W = 64 / TA_P_SPLIT;  // TMEM columns (bf16 pairs) per part
            const int k = (c + 1) / (4 / TA_P_SPLIT) - 1;
            if (W == 32) {
              tmem_st32(tP + 32 * k, pk[k]);
            } else {
              uint32_t q16[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) q16[i] = pk[c >> 1][(c & 1) * 16 + i];
              tmem_st16(tP + 16 * c, q16);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(smem_u32(&bars->p_part[t][k]));
          }
        }
      } else {
        // split the exponentials between the MUFU unit and the FMA pipes
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0, x1;
            f2_split(ffma2(f2(__uint_as_float(s[c][2 * i]), __uint_as_float(s[c][2 * i + 1])), sl2x2, negmx2), x0,
                     x1);
            const bool soft = (i % C::POLY_PERIOD) >= C::POLY_PERIOD - C::POLY_PAIRS;
            const float p0 = soft ? exp2_poly(x0) : ex2(x0);
            const float p1 = soft ? exp2_poly(x1) : ex2(x1);
            if (i & 1) lsB = fadd2(lsB, f2(p0, p1));
            else lsA = fadd2(lsA, f2(p0, p1));
            pk[c >> 1][(c & 1) * 16 + i] = pack_bf16(p0, p1);
          }
        }
      }
      float ls0, ls1;
      f2_split(fadd2(lsA, lsB), ls0, ls1);
      l += ls0 + ls1;
      if constexpr (C::SEP_P) {
        if (j > 0) {  // P V_t(j-1) has read the P_t columns
          ok = wait_bar(smem_u32(&bars->pv_done[t]), (j - 1) & 1, abort_flag, p.timeout_ns);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
        }
      }
      if (TA_P_HALVES && !C::SEP_P && C::POLY_PAIRS != 0 && !(tail || diag)) {
        // the split-exponent path stores all of P and releases its parts only here
        tmem_st32(tP, pk[0]);
        tmem_st32(tP + 32, pk[1]);
        tmem_st_wait();
        tc_fence_before();
        for (int k = 0; k < TA_P_SPLIT - 1; ++k) mbar_arrive(smem_u32(&bars->p_part[t][k]));
      } else if (!TA_P_HALVES || C::SEP_P) {
        tmem_st32(tP, pk[0]);
        tmem_st32(tP + 32, pk[1]);
      } else if (TA_P_SPLIT == 2) {
        tmem_st32(tP + 32, pk[1]);
      } else {
        uint32_t q16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) q16[i] = pk[1][16 + i];
        tmem_st16(tP + 48, q16);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->p_full[t]));
    }
    // ---------------------------------------------------------- epilogue
    if (present[t] && ok) {
      ok = wait_bar(smem_u32(&bars->o_full[t]), 0, abort_flag, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (present[t] && ok) {
      tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      if constexpr (VARLEN) {
        // direct row stores (a tile may end inside the sequence)
        uint16_t* orow = p.o + ((size_t)(qstart + row) * p.H + head) * D;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_ld_wait(o);
          if (row < Nq) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float a = (l > 0.f) ? __uint_as_float(o[g * 8 + 2 * e]) * inv : 0.f;
                const float b = (l > 0.f) ? __uint_as_float(o[g * 8 + 2 * e + 1]) * inv : 0.f;
                w[e] = pack_bf16(a, b);
              }
              *reinterpret_cast<uint4*>(orow + cc * 32 + g * 8) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
        if (row < Nq)
          p.lse[(size_t)head * p.total_q + qstart + row] =
              (l > 0.f) ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
      } else {
      uint8_t* stage = smem + C::Q_OFF + t * C::TILE;  // Q_t is no longer read
      // columns [32 cc, 32 cc + 32) of O_t / l -> bf16 -> the swizzled staging tile
      auto emit = [&](int cc, const uint32_t (&o)[32]) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a = (l > 0.f) ? __uint_as_float(o[g * 8 + 2 * e]) * inv : 0.f;
            const float b = (l > 0.f) ? __uint_as_float(o[g * 8 + 2 * e + 1]) * inv : 0.f;
            w[e] = pack_bf16(a, b);
          }
          const int c16 = cc * 4 + g;  // 16-byte chunk within the row
          const int h = c16 >> 3, ch = c16 & 7;
          uint8_t* dst = stage + h * C::HALF + rr * 128 + ((ch ^ (rr & 7)) << 4);
          *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      };
      if constexpr (D == 128) {
        // every column requested before one wait (the scores' registers are
        // free by now): one tensor-memory round trip instead of four
        uint32_t oall[D / 32][32];
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tO + cc * 32, oall[cc]);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) tmem_ld_wait(oall[cc]);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) emit(cc, oall[cc]);
      } else {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_ld_wait(o);
          emit(cc, o);
        }
      }
      if (row < Nq)
        p.lse[(size_t)bh * Nq + row] = (l > 0.f) ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&bars->epi[t]));
      if (warp == 4 + 4 * t && lane == 0) {
        if (wait_bar(smem_u32(&bars->epi[t]), 0, abort_flag, p.timeout_ns)) {
          for (int h = 0; h < D / 64; ++h)
            tma_store_3d(&tmO, sbase + C::Q_OFF + t * C::TILE + h * C::HALF, h * 64, r0[t], bh);
          bulk_commit();
          bulk_wait_read();  // the CTA may exit once the tile has left shared memory
        }
      }
      __syncwarp();
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

// Empty key set: every query row sees nothing -> O = 0, LSE = -inf.
__global__ void fill_empty_kernel(uint16_t* o, float* lse, long long n_rows, int d) {
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i < n_rows * d) o[i] = 0;
  if (i < n_rows) lse[i] = -INFINITY;
}

}  // namespace ta
