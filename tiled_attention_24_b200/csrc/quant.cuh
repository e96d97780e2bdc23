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

__device__ __forceinline__ int8_t q8(float x, float s) {
  int v = __float2int_rn(__fdiv_rn(x, s));
  v = max(-127, min(127, v));
  return (int8_t)v;
}

// One warp per row of D bf16 values (D = 64 or 128).
template <int D>
__global__ void __launch_bounds__(256) quant_int8_rows_kernel(const uint16_t* __restrict__ x, int8_t* __restrict__ xq,
                                                             float* __restrict__ xs, long long rows) {
  constexpr int E = D / 32;  // elements per lane
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint16_t* src = x + row * D + lane * E;
  float v[E];
  if constexpr (E == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(src);
    v[0] = __uint_as_float(w.x << 16);
    v[1] = __uint_as_float(w.x & 0xFFFF0000u);
    v[2] = __uint_as_float(w.y << 16);
    v[3] = __uint_as_float(w.y & 0xFFFF0000u);
  } else {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(src);
    v[0] = __uint_as_float(w << 16);
    v[1] = __uint_as_float(w & 0xFFFF0000u);
  }
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(v[e]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 127.f);
  uint32_t packed = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) packed |= (uint32_t)(uint8_t)q8(v[e], s) << (8 * e);
  if constexpr (E == 4) {
    *reinterpret_cast<uint32_t*>(xq + row * D + lane * E) = packed;
  } else {
    *reinterpret_cast<uint16_t*>(xq + row * D + lane * E) = (uint16_t)packed;
  }
  if (lane == 0) xs[row] = s;
}

// Per-(batch, head) amax, accumulated with an integer atomicMax on the bit
// pattern (valid for non-negative floats) into amax_bits[bh] (zeroed first).
__global__ void __launch_bounds__(256) head_amax_kernel(const uint16_t* __restrict__ x, unsigned* __restrict__ amax_bits,
                                                        long long per_head) {
  const int bh = blockIdx.y;
  const uint16_t* src = x + (long long)bh * per_head;
  float m = 0.f;
  for (long long i = ((long long)blockIdx.x * 256 + threadIdx.x) * 8; i < per_head; i += (long long)gridDim.x * 256 * 8) {
    const uint4 w = *reinterpret_cast<const uint4*>(src + i);
    m = fmaxf(m, fabsf(__uint_as_float(w.x << 16)));
    m = fmaxf(m, fabsf(__uint_as_float(w.x & 0xFFFF0000u)));
    m = fmaxf(m, fabsf(__uint_as_float(w.y << 16)));
    m = fmaxf(m, fabsf(__uint_as_float(w.y & 0xFFFF0000u)));
    m = fmaxf(m, fabsf(__uint_as_float(w.z << 16)));
    m = fmaxf(m, fabsf(__uint_as_float(w.z & 0xFFFF0000u)));
    m = fmaxf(m, fabsf(__uint_as_float(w.w << 16)));
    m = fmaxf(m, fabsf(__uint_as_float(w.w & 0xFFFF0000u)));
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
  for (long long i = ((long long)blockIdx.x * 256 + threadIdx.x) * 8; i < per_head; i += (long long)gridDim.x * 256 * 8) {
    const uint4 w = *reinterpret_cast<const uint4*>(src + i);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    uint32_t out[2] = {0, 0};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t bits = (e & 1) ? (ws[e >> 1] & 0xFFFF0000u) : (ws[e >> 1] << 16);
      out[e >> 2] |= (uint32_t)(uint8_t)q8(__uint_as_float(bits), s) << (8 * (e & 3));
    }
    *reinterpret_cast<uint2*>(dst + i) = make_uint2(out[0], out[1]);
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

}  // namespace ta
