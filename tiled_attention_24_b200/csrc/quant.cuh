// Quantisers for the low-precision forwards.
//
// INT8 ("INT-FlashAttention" page: token-level post-training quantisation of
// Q, K and V so that the forward's matmuls run as INT8 GEMMs): symmetric, one
// fp32 scale s = amax / 127 per token row (Q, K) or per (batch, head) (V, whose
// P V product contracts over tokens, so its scale must be shared by all tokens
// of a head), q = clamp(rne(x / s), -127, 127), amax = 0 -> s = 1.  Divides are
// IEEE round-to-nearest (__fdiv_rn) so that the result is bit-identical to any
// other correctly rounded fp32 implementation.
#pragma once
#include "ptx.cuh"

namespace ta {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

template <int QMAX = 127>
__device__ __forceinline__ int8_t q8(float x, float s) {
  int v = __float2int_rn(__fdiv_rn(x, s));
  v = max(-QMAX, min(QMAX, v));
  return (int8_t)v;
}

// Row quantiser: LPR = D / 8 lanes per row (16 bytes = 8 bf16 each; 16 lanes
// at d = 128, 8 at d = 64), 32 / LPR rows per warp pass, QROW_PASSES passes
// per warp whose loads are all issued before any row is quantised (bytes in
// flight per lane: 16 x QROW_PASSES).  QMAX = 127 (INT8) or 7 (INT4 codes in
// int8 containers: the same token-level scheme at 4 bits).
constexpr int QROW_PASSES = 4;
template <int D>
__host__ __device__ constexpr long long qrow_rows_per_block() { return 8LL * (32 / (D / 8)) * QROW_PASSES; }

__device__ __forceinline__ void unpack_bf16x8(const uint4& w, float (&v)[8]) {
  v[0] = __uint_as_float(w.x << 16); v[1] = __uint_as_float(w.x & 0xFFFF0000u);
  v[2] = __uint_as_float(w.y << 16); v[3] = __uint_as_float(w.y & 0xFFFF0000u);
  v[4] = __uint_as_float(w.z << 16); v[5] = __uint_as_float(w.z & 0xFFFF0000u);
  v[6] = __uint_as_float(w.w << 16); v[7] = __uint_as_float(w.w & 0xFFFF0000u);
}

template <int D, int QMAX = 127>
__global__ void __launch_bounds__(256) quant_int8_rows_kernel(const uint16_t* __restrict__ x, int8_t* __restrict__ xq,
                                                             float* __restrict__ xs, long long rows) {
  constexpr int LPR = D / 8, RPW = 32 / LPR;
  const int lane = threadIdx.x & 31, sub = lane / LPR, cl = lane % LPR;
  const long long row0 = ((long long)blockIdx.x * 8 + (threadIdx.x >> 5)) * (RPW * QROW_PASSES);
  uint4 w[QROW_PASSES];
#pragma unroll
  for (int pss = 0; pss < QROW_PASSES; ++pss) {
    const long long row = row0 + pss * RPW + sub;
    w[pss] = (row < rows) ? *reinterpret_cast<const uint4*>(x + row * D + cl * 8) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int pss = 0; pss < QROW_PASSES; ++pss) {
    const long long row = row0 + pss * RPW + sub;
    float v[8];
    unpack_bf16x8(w[pss], v);
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = (amax == 0.f) ? 1.f : __fdiv_rn(amax, (float)QMAX);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      lo |= (uint32_t)(uint8_t)q8<QMAX>(v[e], s) << (8 * e);
      hi |= (uint32_t)(uint8_t)q8<QMAX>(v[e + 4], s) << (8 * e);
    }
    if (row < rows) {
      *reinterpret_cast<uint2*>(xq + row * D + cl * 8) = make_uint2(lo, hi);
      if (cl == 0) xs[row] = s;
    }
  }
}

// Per-(batch, head) amax, accumulated with an integer atomicMax on the bit
// pattern (valid for non-negative floats) into amax_bits[bh] (zeroed first).
// Each thread keeps HEAD_UNROLL 16-byte loads in flight.
constexpr int HEAD_UNROLL = 4;
__device__ __forceinline__ float amax_bf16x8(const uint4& w, float m) {
  m = fmaxf(m, fabsf(__uint_as_float(w.x << 16)));
  m = fmaxf(m, fabsf(__uint_as_float(w.x & 0xFFFF0000u)));
  m = fmaxf(m, fabsf(__uint_as_float(w.y << 16)));
  m = fmaxf(m, fabsf(__uint_as_float(w.y & 0xFFFF0000u)));
  m = fmaxf(m, fabsf(__uint_as_float(w.z << 16)));
  m = fmaxf(m, fabsf(__uint_as_float(w.z & 0xFFFF0000u)));
  m = fmaxf(m, fabsf(__uint_as_float(w.w << 16)));
  m = fmaxf(m, fabsf(__uint_as_float(w.w & 0xFFFF0000u)));
  return m;
}
__global__ void __launch_bounds__(256) head_amax_kernel(const uint16_t* __restrict__ x, unsigned* __restrict__ amax_bits,
                                                        long long per_head) {
  const int bh = blockIdx.y;
  const uint16_t* src = x + (long long)bh * per_head;
  const long long stride = (long long)gridDim.x * 256 * 8;
  float m = 0.f;
  for (long long i0 = ((long long)blockIdx.x * 256 + threadIdx.x) * 8; i0 < per_head; i0 += HEAD_UNROLL * stride) {
    uint4 w[HEAD_UNROLL];
#pragma unroll
    for (int u = 0; u < HEAD_UNROLL; ++u) {
      const long long i = i0 + u * stride;
      w[u] = (i < per_head) ? *reinterpret_cast<const uint4*>(src + i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < HEAD_UNROLL; ++u) m = amax_bf16x8(w[u], m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = wm[0];
    for (int w = 1; w < 8; ++w) r = fmaxf(r, wm[w]);
    atomicMax(amax_bits + bh, __float_as_uint(r));
  }
}

__global__ void __launch_bounds__(256) quant_int8_heads_kernel(const uint16_t* __restrict__ x, int8_t* __restrict__ xq,
                                                               const unsigned* __restrict__ amax_bits,
                                                               long long per_head) {
  const int bh = blockIdx.y;
  const float amax = __uint_as_float(amax_bits[bh]);
  const float s = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 127.f);
  const uint16_t* src = x + (long long)bh * per_head;
  int8_t* dst = xq + (long long)bh * per_head;
  const long long stride = (long long)gridDim.x * 256 * 8;
  for (long long i0 = ((long long)blockIdx.x * 256 + threadIdx.x) * 8; i0 < per_head; i0 += HEAD_UNROLL * stride) {
    uint4 w[HEAD_UNROLL];
#pragma unroll
    for (int u = 0; u < HEAD_UNROLL; ++u) {
      const long long i = i0 + u * stride;
      w[u] = (i < per_head) ? *reinterpret_cast<const uint4*>(src + i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < HEAD_UNROLL; ++u) {
      const long long i = i0 + u * stride;
      const uint32_t ws[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
      uint32_t out[2] = {0, 0};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t bits = (e & 1) ? (ws[e >> 1] & 0xFFFF0000u) : (ws[e >> 1] << 16);
        out[e >> 2] |= (uint32_t)(uint8_t)q8(__uint_as_float(bits), s) << (8 * (e & 3));
      }
      if (i < per_head) *reinterpret_cast<uint2*>(dst + i) = make_uint2(out[0], out[1]);
    }
  }
}

// amax bits -> scale, in place (runs after the quantise pass on the same stream).
__global__ void head_scale_kernel(unsigned* amax_bits, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float amax = __uint_as_float(amax_bits[i]);
  const float s = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 127.f);
  amax_bits[i] = __float_as_uint(s);
}

// ---------------------------------------------------------------------------
// NVFP4 ("Hardware-Aware FP4 FlashAttention-4" page: FP4 operands): blocks of
// 16 elements, e2m1 codes (RNE, saturating at +-6) scaled by one unsigned
// e4m3 factor per block, sf = e4m3_rne(amax / 6), code = e2m1_rne(x / sf),
// both divides IEEE fp32.  Negative values that round to zero keep code 0.
//
// Scale factors are stored in the layout the tensor core reads them in: per
// 128-row tile and per group of 4 consecutive blocks (one 64-element MMA
// step), 512 bytes with byte (r % 32) * 16 + (r / 32) * 4 + block % 4 for row
// r of the tile; a 128 x 128 tile has two such groups (1 KB).
// mode 0 (Q, K): blocks along d, codes [BH][N][64 B], sf [BH][ceil(N/128)][1 KB]
// mode 1 (V):    blocks along tokens, written transposed: codes [BH][128][KT*64 B]
//                and sf [BH][KT][1 KB] with KT = ceil(N/128); rows = channels.
// Rows / tokens past N are zero (codes 0, scale 0).

__device__ __forceinline__ uint32_t e4m3_rne(float v) {  // v >= 0, saturating
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.f), "f"(v));
  return r & 0xFFu;
}
__device__ __forceinline__ float e4m3_value(uint32_t c) {  // from the format definition
  const uint32_t e = (c >> 3) & 0xFu, m = c & 7u;
  return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0x1p-9f;
}
// two fp32 -> e2m1 codes, `lo` in the low nibble; negative zero -> code 0
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  if ((r & 0xFu) == 8u) r &= 0xF0u;
  if ((r >> 4) == 8u) r &= 0x0Fu;
  return r;
}
__device__ __forceinline__ uint32_t sf_offset(int r, int blk) {  // within a 1 KB tile
  return (uint32_t)((blk >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (blk & 3));
}
// quantise 16 values; returns the scale code, fills 8 code bytes
__device__ __forceinline__ uint32_t nvfp4_block(const float (&v)[16], uint32_t (&out)[2]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t sfc = e4m3_rne(__fdiv_rn(amax, 6.f));
  const float s = e4m3_value(sfc);
  out[0] = out[1] = 0u;
  if (s > 0.f) {
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const uint32_t b = e2m1x2(__fdiv_rn(v[i], s), __fdiv_rn(v[i + 1], s));
      out[i >> 3] |= b << (8 * ((i >> 1) & 3));
    }
  }
  return sfc;
}

// mode 0: one thread per (bh, padded row, block of 16 along d = 128)
__global__ void __launch_bounds__(256) quant_nvfp4_rows_kernel(const uint16_t* __restrict__ x, uint8_t* __restrict__ codes,
                                                               uint8_t* __restrict__ sf, int N, int RT, long long total) {
  const long long i = (long long)blockIdx.x * 256 + threadIdx.x;
  if (i >= total) return;
  const int blk = (int)(i & 7);
  const long long rowg = i >> 3;              // bh * RT*128 + row
  const int row = (int)(rowg % (RT * 128));
  const long long bh = rowg / (RT * 128);
  float v[16];
  if (row < N) {
    const uint16_t* src = x + ((bh * N + row) * 128 + blk * 16);
    const uint4 w0 = *reinterpret_cast<const uint4*>(src), w1 = *reinterpret_cast<const uint4*>(src + 8);
    const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      v[2 * e] = __uint_as_float(ws[e] << 16);
      v[2 * e + 1] = __uint_as_float(ws[e] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = 0.f;
  }
  uint32_t out[2];
  const uint32_t sfc = nvfp4_block(v, out);
  if (row < N) *reinterpret_cast<uint2*>(codes + (bh * N + row) * 64 + blk * 8) = make_uint2(out[0], out[1]);
  sf[((bh * RT + row / 128) * 1024) + sf_offset(row & 127, blk)] = (uint8_t)sfc;
}

// mode 1: one thread per (bh, token block of 16, channel); consecutive threads
// take consecutive channels so the loads are coalesced
__global__ void __launch_bounds__(256) quant_nvfp4_cols_kernel(const uint16_t* __restrict__ x, uint8_t* __restrict__ codes,
                                                               uint8_t* __restrict__ sf, int N, int KT, long long total) {
  const long long i = (long long)blockIdx.x * 256 + threadIdx.x;
  if (i >= total) return;
  const int c = (int)(i & 127);
  const long long rest = i >> 7;
  const int tb = (int)(rest % (KT * 8));
  const long long bh = rest / (KT * 8);
  float v[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int tok = tb * 16 + e;
    v[e] = (tok < N) ? __uint_as_float((uint32_t)x[(bh * N + tok) * 128 + c] << 16) : 0.f;
  }
  uint32_t out[2];
  const uint32_t sfc = nvfp4_block(v, out);
  *reinterpret_cast<uint2*>(codes + (bh * 128 + c) * (long long)(KT * 64) + tb * 8) = make_uint2(out[0], out[1]);
  sf[((bh * KT + tb / 8) * 1024) + sf_offset(c, tb & 7)] = (uint8_t)sfc;
}

// ---------------------------------------------------------------------------
// FP8 e4m3 with incoherent processing ("Can a full-day context beat one
// minute? ..." page, FA3 list item 3: rotate the vectors before quantising so
// that outliers spread over the coordinates).  Q, K rows: optional rotation
// y = H_d (sigma o x) by the unnormalised fast Walsh-Hadamard transform in
// fp32 (stages h = 1, 2, ..., d/2; (a, b) -> (a + b, a - b)), then one scale
// per row s = amax / 448 and codes e4m3_rne_satfinite(y / s) (IEEE divides).
// V: one scale per (batch, head, channel) over the head's tokens.
__device__ __forceinline__ uint32_t e4m3x2_bits(float lo, float hi) {  // lo -> low byte
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Same lane layout as the INT8 row quantiser: D / 8 lanes per row, 8 values
// per lane (element e = lane_in_row * 8 + i), QROW_PASSES rows per lane with
// all loads issued first.  The transform stages h = 1, 2, 4 run inside a lane,
// h >= 8 across lanes (partner lane differs in bit h / 8), with the same fp32
// operations in the same order as the stage definition.
template <int D>
__global__ void __launch_bounds__(256) quant_fp8_rows_kernel(const uint16_t* __restrict__ x,
                                                             const float* __restrict__ signs,
                                                             uint8_t* __restrict__ codes, float* __restrict__ xs,
                                                             long long rows) {
  constexpr int E = 8, LPR = D / 8, RPW = 32 / LPR;
  const int lane = threadIdx.x & 31, sub = lane / LPR, cl = lane % LPR;
  const long long row0 = ((long long)blockIdx.x * 8 + (threadIdx.x >> 5)) * (RPW * QROW_PASSES);
  float sg[E];
#pragma unroll
  for (int i = 0; i < E; ++i) sg[i] = (signs != nullptr) ? signs[cl * E + i] : 1.f;
  uint4 w[QROW_PASSES];
#pragma unroll
  for (int pss = 0; pss < QROW_PASSES; ++pss) {
    const long long row = row0 + pss * RPW + sub;
    w[pss] = (row < rows) ? *reinterpret_cast<const uint4*>(x + row * D + cl * E) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int pss = 0; pss < QROW_PASSES; ++pss) {
    const long long row = row0 + pss * RPW + sub;
    float v[E];
    unpack_bf16x8(w[pss], v);
    if (signs != nullptr) {
#pragma unroll
      for (int i = 0; i < E; ++i) v[i] *= sg[i];
      // stages inside a lane
#pragma unroll
      for (int h = 1; h < E; h <<= 1) {
#pragma unroll
        for (int i = 0; i < E; ++i) {
          if ((i & h) == 0) {
            const float a = v[i], b = v[i + h];
            v[i] = a + b;
            v[i + h] = a - b;
          }
        }
      }
      // stages across the lanes of the row: partner lane differs in bit h / E
#pragma unroll
      for (int h = E; h < D; h <<= 1) {
        const int lm = h / E;
        const bool upper = (cl & lm) != 0;
#pragma unroll
        for (int i = 0; i < E; ++i) {
          const float o = __shfl_xor_sync(0xffffffffu, v[i], lm);
          v[i] = upper ? (o - v[i]) : (v[i] + o);
        }
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < E; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 448.f);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
      lo |= e4m3x2_bits(__fdiv_rn(v[i], s), __fdiv_rn(v[i + 1], s)) << (8 * i);
      hi |= e4m3x2_bits(__fdiv_rn(v[i + 4], s), __fdiv_rn(v[i + 5], s)) << (8 * i);
    }
    if (row < rows) {
      *reinterpret_cast<uint2*>(codes + row * D + cl * E) = make_uint2(lo, hi);
      if (cl == 0) xs[row] = s;
    }
  }
}

// V: one scale per (batch, head, channel) over the head's tokens.  Three
// passes over chunks of 128 tokens (grid: chunks x BH): per-channel amax
// (atomicMax on the bit patterns of non-negative floats, into the scale
// buffer), codes (each block derives the scales from the amax), then the
// amax words become the scales in place.  A thread covers 8 channels (16 B).
template <int D>
__global__ void __launch_bounds__(256) channel_amax_kernel(const uint16_t* __restrict__ x,
                                                           unsigned* __restrict__ amax_bits, int N) {
  constexpr int G = D / 8, R = 256 / G, PASSES = 128 / R;  // channel groups, token rows per pass
  const int bh = blockIdx.y, g = threadIdx.x % G, r = threadIdx.x / G;
  const int n0 = blockIdx.x * 128, n1 = min(N, n0 + 128);
  const uint16_t* src = x + ((size_t)bh * N) * D + g * 8;
  uint4 w[PASSES];  // every load of the thread in flight at once
#pragma unroll
  for (int k = 0; k < PASSES; ++k) {
    const int n = n0 + r + k * R;
    w[k] = (n < n1) ? *reinterpret_cast<const uint4*>(src + (size_t)n * D) : make_uint4(0, 0, 0, 0);
  }
  float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int k = 0; k < PASSES; ++k) {
    const uint32_t u[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m[2 * i] = fmaxf(m[2 * i], fabsf(__uint_as_float(u[i] << 16)));
      m[2 * i + 1] = fmaxf(m[2 * i + 1], fabsf(__uint_as_float(u[i] & 0xFFFF0000u)));
    }
  }
  __shared__ float part[R][D];
#pragma unroll
  for (int i = 0; i < 8; ++i) part[r][g * 8 + i] = m[i];
  __syncthreads();
  if (threadIdx.x < D) {
    float a = 0.f;
    for (int k = 0; k < R; ++k) a = fmaxf(a, part[k][threadIdx.x]);
    atomicMax(amax_bits + (size_t)bh * D + threadIdx.x, __float_as_uint(a));
  }
}

template <int D>
__global__ void __launch_bounds__(256) channel_codes_kernel(const uint16_t* __restrict__ x,
                                                            const unsigned* __restrict__ amax_bits,
                                                            uint8_t* __restrict__ codes, int N) {
  constexpr int G = D / 8, R = 256 / G, PASSES = 128 / R;
  const int bh = blockIdx.y, g = threadIdx.x % G, r = threadIdx.x / G;
  const int n0 = blockIdx.x * 128, n1 = min(N, n0 + 128);
  const uint16_t* src = x + ((size_t)bh * N) * D + g * 8;
  uint8_t* dst = codes + ((size_t)bh * N) * D + g * 8;
  uint4 w[PASSES];
#pragma unroll
  for (int k = 0; k < PASSES; ++k) {
    const int n = n0 + r + k * R;
    w[k] = (n < n1) ? *reinterpret_cast<const uint4*>(src + (size_t)n * D) : make_uint4(0, 0, 0, 0);
  }
  float sc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float a = __uint_as_float(amax_bits[(size_t)bh * D + g * 8 + i]);
    sc[i] = (a == 0.f) ? 1.f : __fdiv_rn(a, 448.f);
  }
#pragma unroll
  for (int k = 0; k < PASSES; ++k) {
    const int n = n0 + r + k * R;
    const uint32_t u[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
    uint32_t out[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t pr = e4m3x2_bits(__fdiv_rn(__uint_as_float(u[i] << 16), sc[2 * i]),
                                      __fdiv_rn(__uint_as_float(u[i] & 0xFFFF0000u), sc[2 * i + 1]));
      if (i & 1)
        out[i >> 1] |= pr << 16;
      else
        out[i >> 1] = pr;
    }
    if (n < n1) *reinterpret_cast<uint2*>(dst + (size_t)n * D) = make_uint2(out[0], out[1]);
  }
}

__global__ void channel_scale_kernel(unsigned* amax_bits, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float amax = __uint_as_float(amax_bits[i]);
  amax_bits[i] = __float_as_uint((amax == 0.f) ? 1.f : __fdiv_rn(amax, 448.f));
}

}  // namespace ta
