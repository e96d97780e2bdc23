// Split-KV decode: one query row per (batch, head) against a long KV cache.
//
// Decode reads every cached key and value once and does ~1 FLOP per byte, so
// it is bound by HBM bandwidth, not by the tensor cores.  The key range of each
// (batch, head) is cut into `num_splits` chunks so that the whole GPU streams
// the cache in parallel; each chunk yields a partial result (O_c, LSE_c) and a
// second, tiny kernel merges them with LSE weights -- the same identity as the
// online-softmax recurrence ("Can a full-day context beat one minute? Flash
// attention and the sequence-length question", section "Online softmax
// recurrence"), applied once to whole chunks.
//
// Split kernel: one 128-thread CTA per (batch*head, chunk), consecutive CTAs
// read consecutive memory; with grouped-query attention the query heads of a
// group are consecutive too, so their shared cache is read from HBM once and
// from L2 by the rest of the group.  A chunk is processed in sub-blocks of 512 keys:
//   1. scores: D/8 lanes per key, each lane a 16-byte slice of the key row
//      (coalesced 16-byte non-allocating loads, 8 in flight per lane), lane
//      partial dot products reduced with warp shuffles; x = score*scale*log2e
//      kept in shared memory;
//   2. running max / rescale / exp2 / row sum over the sub-block;
//   3. values: same lane layout over V rows, fp32 accumulators per lane.
// Partial O_c (normalised) and LSE_c go to the caller's workspace.
#pragma once
#include "ptx.cuh"

namespace ta {

constexpr int DEC_THREADS = 128;
constexpr int DEC_SB = 512;  // keys per sub-block
constexpr int DEC_UNROLL = 8;
// grouped kernel: loads in flight per lane, by heads per CTA (measured on
// B200 with B64 Hq32 N_kv 8192, G = 4: 0.499 ms with 8, 0.516 with 4,
// 1.07 with 2; G = 8 also fastest with 8)
__host__ __device__ constexpr int dec_group_unroll(int) { return 8; }

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int D>
__global__ void __launch_bounds__(DEC_THREADS)
    decode_split_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                        const uint16_t* __restrict__ v, float* __restrict__ o_part,
                        float* __restrict__ lse_part, int Nkv, int S, int chunk, float sl2, int group,
                        const int* __restrict__ seqlens, int Hq) {
  constexpr int LPK = D / 8;          // lanes per key row (16 bytes each)
  constexpr int KPW = 32 / LPK;       // key rows per warp step
  constexpr int NW = DEC_THREADS / 32;
  constexpr int PER_WARP = DEC_SB / NW;
  constexpr int STEPS = PER_WARP / (KPW * DEC_UNROLL);
  static_assert(PER_WARP % (KPW * DEC_UNROLL) == 0, "sub-block split");

  __shared__ float xs[DEC_SB];
  __shared__ float red[NW][D];
  __shared__ float wred[NW];

  const int bh = blockIdx.x / S, c = blockIdx.x % S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPK;                    // which key of the warp step
  const int e0 = (lane % LPK) * 8;               // first channel of this lane
  // per-batch cache length (seqlens != null): keys [0, len) of the Nkv rows
  const int len = seqlens ? min(max(seqlens[bh / Hq], 0), Nkv) : Nkv;
  if (seqlens) chunk = (len + S - 1) / S;
  const long long key0 = (long long)c * chunk;
  const int nk = (int)max(0LL, min((long long)len, key0 + chunk) - key0);

  float qv[8];
  {
    const uint4 w = *reinterpret_cast<const uint4*>(q + (size_t)bh * D + e0);
    qv[0] = bf_lo(w.x); qv[1] = bf_hi(w.x); qv[2] = bf_lo(w.y); qv[3] = bf_hi(w.y);
    qv[4] = bf_lo(w.z); qv[5] = bf_hi(w.z); qv[6] = bf_lo(w.w); qv[7] = bf_hi(w.w);
  }
  const int kvh = bh / group;  // cache head of this query head (grouped-query attention)
  const uint16_t* kb = k + ((size_t)kvh * Nkv + key0) * D + e0;
  const uint16_t* vb = v + ((size_t)kvh * Nkv + key0) * D + e0;

  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

  for (int s0 = 0; s0 < nk; s0 += DEC_SB) {
    const int ns = min(DEC_SB, nk - s0);
    // ---- 1. scores of this sub-block
#pragma unroll 1
    for (int st = 0; st < STEPS; ++st) {
      uint4 kr[DEC_UNROLL];
#pragma unroll
      for (int u = 0; u < DEC_UNROLL; ++u) {
        const int kk = warp * PER_WARP + (st * DEC_UNROLL + u) * KPW + sub;
        kr[u] = (kk < ns) ? ldg_stream(kb + (size_t)(s0 + kk) * D) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < DEC_UNROLL; ++u) {
        float a = qv[0] * bf_lo(kr[u].x);
        a = fmaf(qv[1], bf_hi(kr[u].x), a);
        a = fmaf(qv[2], bf_lo(kr[u].y), a);
        a = fmaf(qv[3], bf_hi(kr[u].y), a);
        a = fmaf(qv[4], bf_lo(kr[u].z), a);
        a = fmaf(qv[5], bf_hi(kr[u].z), a);
        a = fmaf(qv[6], bf_lo(kr[u].w), a);
        a = fmaf(qv[7], bf_hi(kr[u].w), a);
#pragma unroll
        for (int o = LPK / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        const int kk = warp * PER_WARP + (st * DEC_UNROLL + u) * KPW + sub;
        if ((lane % LPK) == 0) xs[kk] = (kk < ns) ? a * sl2 : -INFINITY;
      }
    }
    __syncthreads();
    // ---- 2. sub-block max, rescale, exp2, sum
    float mx = -INFINITY;
    for (int i = threadIdx.x; i < DEC_SB; i += DEC_THREADS) mx = fmaxf(mx, xs[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) wred[warp] = mx;
    __syncthreads();
    mx = wred[0];
#pragma unroll
    for (int w = 1; w < NW; ++w) mx = fmaxf(mx, wred[w]);
    const float m_new = fmaxf(m_run, mx);     // finite: the sub-block has >= 1 key
    const float factor = ex2(m_run - m_new);  // 0 on the first sub-block
    float ps = 0.f;
    for (int i = threadIdx.x; i < DEC_SB; i += DEC_THREADS) {
      const float pv = ex2(xs[i] - m_new);    // -inf -> 0
      xs[i] = pv;
      ps += pv;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
    __syncthreads();  // everyone has read wred (max) before it is reused
    if (lane == 0) wred[warp] = ps;
    __syncthreads();
    float psum = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) psum += wred[w];
    l_run = l_run * factor + psum;
    m_run = m_new;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= factor;
    // ---- 3. values
#pragma unroll 1
    for (int st = 0; st < STEPS; ++st) {
      uint4 vr[DEC_UNROLL];
#pragma unroll
      for (int u = 0; u < DEC_UNROLL; ++u) {
        const int kk = warp * PER_WARP + (st * DEC_UNROLL + u) * KPW + sub;
        vr[u] = (kk < ns) ? ldg_stream(vb + (size_t)(s0 + kk) * D) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < DEC_UNROLL; ++u) {
        const int kk = warp * PER_WARP + (st * DEC_UNROLL + u) * KPW + sub;
        const float pw = xs[kk];  // 0 for keys past the end
        acc[0] = fmaf(pw, bf_lo(vr[u].x), acc[0]);
        acc[1] = fmaf(pw, bf_hi(vr[u].x), acc[1]);
        acc[2] = fmaf(pw, bf_lo(vr[u].y), acc[2]);
        acc[3] = fmaf(pw, bf_hi(vr[u].y), acc[3]);
        acc[4] = fmaf(pw, bf_lo(vr[u].z), acc[4]);
        acc[5] = fmaf(pw, bf_hi(vr[u].z), acc[5]);
        acc[6] = fmaf(pw, bf_lo(vr[u].w), acc[6]);
        acc[7] = fmaf(pw, bf_hi(vr[u].w), acc[7]);
      }
    }
    __syncthreads();  // xs / wred are rewritten by the next sub-block
  }

  // ---- reduce the per-lane accumulators over the KPW key groups and warps
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
  if (sub == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red[warp][e0 + e] = acc[e];
  }
  __syncthreads();
  const size_t part = (size_t)bh * S + c;
  for (int e = threadIdx.x; e < D; e += DEC_THREADS) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) sum += red[w][e];
    o_part[part * D + e] = (nk > 0) ? sum / l_run : 0.f;
  }
  if (threadIdx.x == 0)
    lse_part[part] = (nk > 0) ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
}

// Grouped-query split kernel: one CTA per (G = 2 or 4 consecutive query heads
// that share a cache head, chunk).  Each key and value row is read from memory
// once and used by all G query heads, so the bytes moved per query head drop
// by G ([FA4-overview] "Compatibility and current status": several heads
// share one key/value projection).  Same lane layout and sub-block online
// softmax as decode_split_kernel, with G scores per key.
template <int D, int G, int NT = DEC_THREADS, int UNR = dec_group_unroll(G)>
__global__ void __launch_bounds__(NT)
    decode_split_group_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                              const uint16_t* __restrict__ v, float* __restrict__ o_part,
                              float* __restrict__ lse_part, int Nkv, int S, int chunk, float sl2, int group,
                              const int* __restrict__ seqlens, int Hq) {
  constexpr int LPK = D / 8;
  constexpr int KPW = 32 / LPK;
  constexpr int NW = NT / 32;
  constexpr int PER_WARP = DEC_SB / NW;
  constexpr int STEPS = PER_WARP / (KPW * UNR);
  static_assert(PER_WARP % (KPW * UNR) == 0, "sub-block split");

  __shared__ float xs[G][DEC_SB];
  __shared__ float red[NW][D];
  __shared__ float wred[NW][G];

  const int grp = blockIdx.x / S, c = blockIdx.x % S;
  const int bh0 = grp * G;         // first query head (batch * Hq + head) of this CTA
  const int kvh = bh0 / group;     // their cache head (G divides the group size)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPK;
  const int e0 = (lane % LPK) * 8;
  const int len = seqlens ? min(max(seqlens[bh0 / Hq], 0), Nkv) : Nkv;  // per-batch cache length
  if (seqlens) chunk = (len + S - 1) / S;
  const long long key0 = (long long)c * chunk;
  const int nk = (int)max(0LL, min((long long)len, key0 + chunk) - key0);

  float qv[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 w = *reinterpret_cast<const uint4*>(q + (size_t)(bh0 + g) * D + e0);
    qv[g][0] = bf_lo(w.x); qv[g][1] = bf_hi(w.x); qv[g][2] = bf_lo(w.y); qv[g][3] = bf_hi(w.y);
    qv[g][4] = bf_lo(w.z); qv[g][5] = bf_hi(w.z); qv[g][6] = bf_lo(w.w); qv[g][7] = bf_hi(w.w);
  }
  const uint16_t* kb = k + ((size_t)kvh * Nkv + key0) * D + e0;
  const uint16_t* vb = v + ((size_t)kvh * Nkv + key0) * D + e0;

  float acc[G][8];
  float m_run[G], l_run[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -INFINITY;
    l_run[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
  }

  for (int s0 = 0; s0 < nk; s0 += DEC_SB) {
    const int ns = min(DEC_SB, nk - s0);
    // ---- 1. G scores per key of this sub-block
#pragma unroll 1
    for (int st = 0; st < STEPS; ++st) {
      uint4 kr[UNR];
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int kk = warp * PER_WARP + (st * UNR + u) * KPW + sub;
        kr[u] = (kk < ns) ? ldg_stream(kb + (size_t)(s0 + kk) * D) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int kk = warp * PER_WARP + (st * UNR + u) * KPW + sub;
        const float k0 = bf_lo(kr[u].x), k1 = bf_hi(kr[u].x), k2 = bf_lo(kr[u].y), k3 = bf_hi(kr[u].y);
        const float k4 = bf_lo(kr[u].z), k5 = bf_hi(kr[u].z), k6 = bf_lo(kr[u].w), k7 = bf_hi(kr[u].w);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float a = qv[g][0] * k0;
          a = fmaf(qv[g][1], k1, a);
          a = fmaf(qv[g][2], k2, a);
          a = fmaf(qv[g][3], k3, a);
          a = fmaf(qv[g][4], k4, a);
          a = fmaf(qv[g][5], k5, a);
          a = fmaf(qv[g][6], k6, a);
          a = fmaf(qv[g][7], k7, a);
#pragma unroll
          for (int o = LPK / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
          if ((lane % LPK) == 0) xs[g][kk] = (kk < ns) ? a * sl2 : -INFINITY;
        }
      }
    }
    __syncthreads();
    // ---- 2. per head: sub-block max, rescale, exp2, sum
    float mx[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      mx[g] = -INFINITY;
      for (int i = threadIdx.x; i < DEC_SB; i += NT) mx[g] = fmaxf(mx[g], xs[g][i]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], o));
      if (lane == 0) wred[warp][g] = mx[g];
    }
    __syncthreads();
    float factor[G], ps[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      mx[g] = wred[0][g];
#pragma unroll
      for (int w = 1; w < NW; ++w) mx[g] = fmaxf(mx[g], wred[w][g]);
      const float m_new = fmaxf(m_run[g], mx[g]);  // finite: the sub-block has >= 1 key
      factor[g] = ex2(m_run[g] - m_new);           // 0 on the first sub-block
      m_run[g] = m_new;
      ps[g] = 0.f;
      for (int i = threadIdx.x; i < DEC_SB; i += NT) {
        const float pv = ex2(xs[g][i] - m_new);      // -inf -> 0
        xs[g][i] = pv;
        ps[g] += pv;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps[g] += __shfl_xor_sync(0xffffffffu, ps[g], o);
    }
    __syncthreads();  // everyone has read wred (max) before it is reused
    if (lane == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) wred[warp][g] = ps[g];
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float psum = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) psum += wred[w][g];
      l_run[g] = l_run[g] * factor[g] + psum;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[g][e] *= factor[g];
    }
    // ---- 3. values: each V row once, for all G heads
#pragma unroll 1
    for (int st = 0; st < STEPS; ++st) {
      uint4 vr[UNR];
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int kk = warp * PER_WARP + (st * UNR + u) * KPW + sub;
        vr[u] = (kk < ns) ? ldg_stream(vb + (size_t)(s0 + kk) * D) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int kk = warp * PER_WARP + (st * UNR + u) * KPW + sub;
        const float v0 = bf_lo(vr[u].x), v1 = bf_hi(vr[u].x), v2 = bf_lo(vr[u].y), v3 = bf_hi(vr[u].y);
        const float v4 = bf_lo(vr[u].z), v5 = bf_hi(vr[u].z), v6 = bf_lo(vr[u].w), v7 = bf_hi(vr[u].w);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pw = xs[g][kk];  // 0 for keys past the end
          acc[g][0] = fmaf(pw, v0, acc[g][0]);
          acc[g][1] = fmaf(pw, v1, acc[g][1]);
          acc[g][2] = fmaf(pw, v2, acc[g][2]);
          acc[g][3] = fmaf(pw, v3, acc[g][3]);
          acc[g][4] = fmaf(pw, v4, acc[g][4]);
          acc[g][5] = fmaf(pw, v5, acc[g][5]);
          acc[g][6] = fmaf(pw, v6, acc[g][6]);
          acc[g][7] = fmaf(pw, v7, acc[g][7]);
        }
      }
    }
    __syncthreads();  // xs / wred are rewritten by the next sub-block
  }

  // ---- per head: reduce the per-lane accumulators over key groups and warps
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int o = LPK; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], o);
    if (sub == 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) red[warp][e0 + e] = acc[g][e];
    }
    __syncthreads();
    const size_t part = (size_t)(bh0 + g) * S + c;
    for (int e = threadIdx.x; e < D; e += NT) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) sum += red[w][e];
      o_part[part * D + e] = (nk > 0) ? sum / l_run[g] : 0.f;
    }
    if (threadIdx.x == 0)
      lse_part[part] = (nk > 0) ? (m_run[g] + log2f(l_run[g])) * 0.69314718055994531f : -INFINITY;
    __syncthreads();  // red is rewritten for the next head
  }
}

// Merge: LSE = log sum_c exp(LSE_c), O = sum_c exp(LSE_c - LSE) O_c -> bf16.
template <int D>
__global__ void __launch_bounds__(D)
    decode_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                          uint16_t* __restrict__ o, float* __restrict__ lse, int S) {
  const int bh = blockIdx.x, e = threadIdx.x;
  const float* lp = lse_part + (size_t)bh * S;
  float mx = -INFINITY;
  for (int c = 0; c < S; ++c) mx = fmaxf(mx, lp[c]);
  const float L2E = 1.4426950408889634f;
  float tot = 0.f, acc = 0.f;
  if (mx != -INFINITY) {
    for (int c = 0; c < S; ++c) {
      const float w = ex2((lp[c] - mx) * L2E);
      tot += w;
      acc = fmaf(w, o_part[((size_t)bh * S + c) * D + e], acc);
    }
  }
  const float out = (mx != -INFINITY) ? acc / tot : 0.f;
  const uint32_t b = pack_bf16(out, 0.f);
  o[(size_t)bh * D + e] = (uint16_t)(b & 0xFFFFu);
  if (e == 0) lse[bh] = (mx != -INFINITY) ? mx + logf(tot) : -INFINITY;
}

}  // namespace ta
