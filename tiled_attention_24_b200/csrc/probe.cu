// Throughput microbenchmarks for the roofline denominators (see
// include/tiledattn_probe.h).  Built as its own library, libtiledattn_probe.so;
// nothing in the attention path calls it.
//
// tap_mma_rate: one CTA per SM issues back-to-back tcgen05.mma from shared
// memory into one tensor-memory accumulator, with the operand layouts the
// attention kernels use (128-byte swizzled K-major tiles for bf16 / int8 /
// e4m3, 64-byte swizzled for e2m1 with ue4m3 scale factors copied into tensor
// memory by tcgen05.cp).  The issuing thread reads %clock64 before the first
// MMA and after the commit barrier of the last one completes.
#include <cstdint>

#include <cuda_runtime.h>

#include "ptx.cuh"
#include "tiledattn_probe.h"

#define TAP_API extern "C" __attribute__((visibility("default")))

namespace tap {

using namespace ta;

constexpr int kMmaSmem = 160 * 1024;  // more than half an SM's shared memory: one CTA per SM

__host__ __device__ constexpr uint32_t idesc_mn(uint32_t fmt_bits, int N) {
  return fmt_bits | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
// D / A / B format fields of the instruction descriptor per kind
constexpr uint32_t kFmtBf16 = (1u << 4) | (1u << 7) | (1u << 10);  // D f32, A bf16, B bf16
constexpr uint32_t kFmtI8 = (2u << 4) | (1u << 7) | (1u << 10);    // D s32, A s8, B s8
constexpr uint32_t kFmtF8 = (1u << 4);                             // D f32, A e4m3, B e4m3
constexpr uint32_t kFmtF4 = (1u << 7) | (1u << 10);                // A e2m1, B e2m1, scales ue4m3

__device__ __forceinline__ void mma_kind(int kind, uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc,
                                         uint32_t sfa, uint32_t sfb) {
  switch (kind) {
    case TAP_KIND_BF16:
      mma_f16_ss(d, a, b, id, acc);
      break;
    case TAP_KIND_I8:
      asm volatile(
          "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
          "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
          "l"(a), "l"(b), "r"(id), "r"(acc)
          : "memory");
      break;
    case TAP_KIND_F8:
      asm volatile(
          "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
          "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
          "l"(a), "l"(b), "r"(id), "r"(acc)
          : "memory");
      break;
    default:
      asm volatile(
          "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
          "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], "
          "p;\n\t}" ::"r"(d),
          "l"(a), "l"(b), "r"(id), "r"(sfa), "r"(sfb), "r"(acc)
          : "memory");
      break;
  }
}

// A operand from tensor memory (bf16, int8, e4m3 kinds)
__device__ __forceinline__ void mma_kind_ts(int kind, uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t id,
                                            uint32_t acc) {
  switch (kind) {
    case TAP_KIND_BF16:
      mma_f16_ts(d, a_tmem, b, id, acc);
      break;
    case TAP_KIND_I8:
      asm volatile(
          "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
          "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
          "r"(a_tmem), "l"(b), "r"(id), "r"(acc)
          : "memory");
      break;
    default:
      asm volatile(
          "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
          "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
          "r"(a_tmem), "l"(b), "r"(id), "r"(acc)
          : "memory");
      break;
  }
}

__device__ __forceinline__ uint64_t desc_layout(uint32_t saddr, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(16u >> 4) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)layout << 61;
  return d;
}

// A finite operand byte pattern per kind (values in [-1, 1] for bf16, no
// NaN codes for e4m3; int8 and e2m1 codes are all finite).
__device__ __forceinline__ uint32_t fill_word(int kind, uint32_t i) {
  uint32_t h = i * 2654435761u;
  h ^= h >> 15;
  h *= 2246822519u;
  h ^= h >> 13;
  if (kind == TAP_KIND_BF16) {
    // two bf16 with exponent 0x70..0x7E (|x| in [2^-15, 1)), random sign / mantissa
    const uint32_t lo = (h & 0x807Fu) | ((0x70u + (h >> 8) % 15u) << 7);
    const uint32_t hi = ((h >> 16) & 0x807Fu) | ((0x70u + (h >> 24) % 15u) << 7);
    return lo | (hi << 16);
  }
  if (kind == TAP_KIND_F8) return h & 0xF7F7F7F7u;  // exponent field <= 14 in every byte
  return h;
}

__global__ void __launch_bounds__(128, 1) mma_loop_kernel(int kind, int n, int iters, int flags,
                                                          unsigned long long* cycles) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // layout: A tile [0, 16 KB), B tile [16 KB, 16 KB + n * 128), scales (1 KB) after, barrier after that
  const bool f4 = (kind == TAP_KIND_F4);
  const int row_bytes = f4 ? 64 : 128;
  const int a_bytes = 128 * row_bytes, b_bytes = n * row_bytes;
  const int sf_off = a_bytes + b_bytes;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + sf_off + 1024);  // [2]: one per issuing thread
  uint32_t* tbase_slot = reinterpret_cast<uint32_t*>(smem + sf_off + 1024 + 16);
  int* abort_flag = reinterpret_cast<int*>(smem + sf_off + 1024 + 20);
  const bool a_tmem = (flags & TAP_A_TMEM) != 0, two_acc = (flags & TAP_TWO_ACC) != 0;
  const int issuers = (flags & TAP_TWO_ISSUERS) ? 2 : 1;
  const uint32_t sbase = smem_u32(smem);

  uint32_t* w = reinterpret_cast<uint32_t*>(smem);
  for (int i = threadIdx.x; i < (a_bytes + b_bytes) / 4; i += blockDim.x)
    w[i] = fill_word(kind, (uint32_t)i + 7919u * blockIdx.x);
  for (int i = threadIdx.x; i < 256; i += blockDim.x)
    reinterpret_cast<uint32_t*>(smem + sf_off)[i] = 0x38383838u;  // ue4m3 1.0
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar[0]), 1);
    mbar_init(smem_u32(&bar[1]), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  fence_proxy_async_smem();  // the tensor core reads these bytes through the async proxy
  if (threadIdx.x < 32) {
    tmem_alloc(smem_u32(tbase_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tbase_slot;
  // A operand in tensor memory (columns [256, 288): 128 lanes x 32 x 32 bit =
  // the 128 bytes of K of the four MMAs), written by the four warps (each
  // its lane quarter) from the same finite pattern
  constexpr uint32_t kTA = 256;
  if (a_tmem) {
    const int wq = threadIdx.x >> 5;
    uint32_t r[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) r[c] = fill_word(kind, (uint32_t)(threadIdx.x * 32 + c));
    tmem_st32(tbase + ((uint32_t)(wq * 32) << 16) + kTA, r);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int wi = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0 && wi < issuers) {
    const uint32_t layout = f4 ? 4u : 2u, sbo = f4 ? 512u : 1024u;
    const uint64_t da = desc_layout(sbase, sbo, layout);
    const uint64_t db = desc_layout(sbase + a_bytes, sbo, layout);
    uint32_t id;
    switch (kind) {
      case TAP_KIND_BF16: id = idesc_mn(kFmtBf16, n); break;
      case TAP_KIND_I8: id = idesc_mn(kFmtI8, n); break;
      case TAP_KIND_F8: id = idesc_mn(kFmtF8, n); break;
      default: id = idesc_mn(kFmtF4, n); break;
    }
    // scale factors: columns [256, 272) for A and [272, 288) for B
    const uint32_t t_sfa = tbase + 256, t_sfb = tbase + 272;
    if (f4) {
      const uint64_t dsf = desc_layout(sbase + sf_off, 128, 0);
      for (int c = 0; c < 4; ++c) {
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(t_sfa + 4 * c), "l"(dsf) : "memory");
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(t_sfb + 4 * c), "l"(dsf) : "memory");
      }
    }
    // four MMAs per iteration, each reading 32 bytes of every operand row:
    // 128-byte rows -> the four 32-byte steps of the swizzle atom; 64-byte
    // rows (e2m1) -> its two steps, twice
    // accumulators: D_0 = columns [0, n); the second issuer, or the second of
    // two alternating chains, uses D_1 = [128, 256) (n = 128 only)
    const uint32_t d0 = tbase + (wi == 1 ? 128u : 0u);
    const long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int step = f4 ? (kk & 1) : kk;
        const uint32_t d = (two_acc && (kk & 1)) ? d0 + 128u : d0;
        const uint32_t acc = (it > 0 || kk >= (two_acc ? 2 : 1)) ? 1u : 0u;
        if (a_tmem)
          mma_kind_ts(kind, d, tbase + kTA + 8 * step, db + (uint64_t)(step * 2), id, acc);
        else
          mma_kind(kind, d, da + (uint64_t)(step * 2), db + (uint64_t)(step * 2), id, acc, t_sfa + 4 * step,
                   t_sfb + 4 * step);
      }
    }
    tc_commit(smem_u32(&bar[wi]));
    const bool ok = wait_bar(smem_u32(&bar[wi]), 0, abort_flag, 1000000000ull);
    tc_fence_after();
    const long long t1 = clock64();
    if (wi == 0) cycles[blockIdx.x] = ok ? (unsigned long long)(t1 - t0) : (unsigned long long)(-5LL);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// Straight-line issue: KIND, N and the operand source fixed at compile time,
// descriptors built before the loop, eight MMAs per group with immediate
// offsets (the K = 128 sweep of an attention tile); after each group a
// commit to an mbarrier (COMMIT = 1) as the attention kernels do.
template <int KIND, int N, bool A_TMEM, bool COMMIT, int BMODE, int SYNC = 0>
__global__ void __launch_bounds__(128, 1) mma_tight_kernel(int iters, unsigned long long* cycles) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // A: two 128-row x 128-byte tiles (K = 256 bytes); B: two N-row x 128-byte tiles
  constexpr int A_BYTES = 2 * 128 * 128, B_BYTES = 2 * N * 128;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + A_BYTES + B_BYTES);  // [4]: commit, final 0, completed, final 1
  uint32_t* tbase_slot = reinterpret_cast<uint32_t*>(smem + A_BYTES + B_BYTES + 32);
  int* abort_flag = reinterpret_cast<int*>(smem + A_BYTES + B_BYTES + 36);
  const uint32_t sbase = smem_u32(smem);
  uint32_t* w = reinterpret_cast<uint32_t*>(smem);
  for (int i = threadIdx.x; i < (A_BYTES + B_BYTES) / 4; i += blockDim.x)
    w[i] = fill_word(KIND, (uint32_t)i + 7919u * blockIdx.x);
  // e2m1 scale factors (ue4m3 1.0), 1 KB after the barrier block
  constexpr int SF_OFF = A_BYTES + B_BYTES + 1024;
  if (KIND == TAP_KIND_F4)
    for (int i = threadIdx.x; i < 256; i += blockDim.x) reinterpret_cast<uint32_t*>(smem + SF_OFF)[i] = 0x38383838u;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar[0]), 1);
    mbar_init(smem_u32(&bar[1]), 1);
    mbar_init(smem_u32(&bar[2]), 1);
    mbar_init(smem_u32(&bar[3]), 1);
    *abort_flag = 0;
    fence_mbar_init();
    mbar_arrive(smem_u32(&bar[2]));  // phase 0 of bar[2] completes at once
    abort_flag[1] = 0;
    abort_flag[2] = 1;  // the flag the FLAGPOLL / FLAGFENCE variants load
  }
  fence_proxy_async_smem();
  if (threadIdx.x < 32) {
    tmem_alloc(smem_u32(tbase_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tbase_slot;
  constexpr uint32_t kTA = 256;  // A in TMEM: columns [256, 320) (K = 256 bytes)
  if (A_TMEM) {
    const int wq = threadIdx.x >> 5;
    uint32_t r[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) r[c] = fill_word(KIND, (uint32_t)(threadIdx.x * 32 + c));
    tmem_st32(tbase + ((uint32_t)(wq * 32) << 16) + kTA, r);
    tmem_st32(tbase + ((uint32_t)(wq * 32) << 16) + kTA + 32, r);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if ((SYNC & 4) && threadIdx.x >= 32 && !(SYNC & 8)) {
    // warps 1..3: tensor-memory traffic like the attention softmax (load 128
    // columns, store 64) over columns [384, 512) of their lane quarter, until
    // the issuing thread raises the stop flag (bounded by a time limit)
    const int wq = threadIdx.x >> 5;
    const uint32_t base = tbase + ((uint32_t)(wq * 32) << 16) + 384;
    volatile int* stop = abort_flag + 1;
    const uint64_t t0s = global_ns();
    while (!*stop && global_ns() - t0s < 1000000000ull) {
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(base + 32 * (c & 3), r[c]);
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_wait(r[c]);
#pragma unroll
      for (int i = 0; i < 32; ++i) r[0][i] ^= r[1][i] ^ r[2][i] ^ r[3][i];
      tmem_st32(base, r[0]);
      tmem_st32(base + 32, r[0]);
      tmem_st_wait();
    }
  }
  const int issuer = (SYNC & 8) ? (threadIdx.x >> 5) : 0;
  if ((threadIdx.x & 31) == 0 && ((SYNC & 8) ? issuer < 2 : threadIdx.x == 0)) {
    constexpr uint32_t fmt = (KIND == TAP_KIND_BF16) ? kFmtBf16
                             : (KIND == TAP_KIND_I8)  ? kFmtI8
                             : (KIND == TAP_KIND_F8)  ? kFmtF8
                                                      : kFmtF4;
    constexpr uint32_t id = idesc_mn(fmt, N);
    // e2m1 (block-scaled): 64-byte rows, 64-byte swizzle, four 128 x 64-byte
    // tiles per operand (K = 512 per row), two MMAs (K = 64, 32 bytes) per
    // tile; scale factors in columns [320, 336) (A) and [336, 352) (B)
    const uint32_t t_sfa = tbase + 320, t_sfb = tbase + 336;
    if (KIND == TAP_KIND_F4) {
      const uint64_t dsf = desc_layout(sbase + SF_OFF, 128, 0);
      for (int c = 0; c < 4; ++c) {
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(t_sfa + 4 * c), "l"(dsf) : "memory");
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(t_sfb + 4 * c), "l"(dsf) : "memory");
      }
    }
    const uint64_t da4 = desc_layout(sbase, 512, 4), db4 = desc_layout(sbase + A_BYTES, 512, 4);
    // MN-major B (N contiguous, as the attention kernels read V): the tile is
    // two 64-element-wide halves (bf16; 128 wide for 8-bit) of K rows x 128
    // bytes, LBO = the distance between halves, SBO = 8 rows
    constexpr uint32_t id_mn = id | (1u << 16);
    constexpr int ROWS_PER_MMA = (KIND == TAP_KIND_BF16) ? 16 : 32;  // K per MMA
    const uint64_t da = desc_layout(sbase, 1024, 2);
    const uint64_t db = desc_layout(sbase + A_BYTES, 1024, 2);
    uint64_t db_mn = desc_layout(sbase + A_BYTES, 1024, 2);
    db_mn |= (uint64_t)((16384u >> 4) & 0x3FFFu) << 16;  // LBO = 16 KB
    const uint32_t cb = smem_u32(&bar[0]);
    const uint32_t done_bar = smem_u32(&bar[2]);
    bool seen = true;
    const long long t0 = clock64();
    const uint32_t flag_addr = smem_u32(abort_flag + 2);  // a word set to 1 before the loop
    auto flag_acquire = [&]() -> uint32_t {
      uint32_t v;
      asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(flag_addr) : "memory");
      return v;
    };
    for (int it = 0; it < iters; ++it) {
      if (SYNC & 2) {  // between groups: a wait on a completed barrier, then the tcgen05 fence
        seen = seen && wait_bar(done_bar, 0, abort_flag, 1000000000ull);
        tc_fence_after();
      }
      if (SYNC & 32) {  // between groups: an acquire load of a set flag, then the tcgen05 fence
        seen = (flag_acquire() != 0u) && seen;
        tc_fence_after();
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        if ((SYNC & 1) && kk == 7) seen = mbar_test_wait(done_bar, 0) && seen;
        if ((SYNC & 16) && kk == 7) seen = (flag_acquire() != 0u) && seen;
        // 32 bytes of K per MMA: step kk & 3 inside a 128-byte atom, atom kk >> 2
        const uint64_t ao = (uint64_t)(((kk >> 2) * 128 * 128 + (kk & 3) * 32) >> 4);
        const uint64_t bo = (uint64_t)(((kk >> 2) * N * 128 + (kk & 3) * 32) >> 4);
        const uint64_t bo_mn = (uint64_t)((kk * ROWS_PER_MMA * 128) >> 4);
        const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
        if (KIND == TAP_KIND_F4) {
          const uint64_t ao4 = (uint64_t)(((kk >> 1) * 128 * 64 + (kk & 1) * 32) >> 4);
          const uint64_t bo4 = (uint64_t)(((kk >> 1) * N * 64 + (kk & 1) * 32) >> 4);
          mma_kind(KIND, tbase, da4 + ao4, db4 + bo4, id, acc, t_sfa + 4 * (kk & 1), t_sfb + 4 * (kk & 1));
        } else if (BMODE == 0) {
          if (A_TMEM)
            mma_kind_ts(KIND, tbase, tbase + kTA + 8 * kk, db + bo, id, acc);
          else
            mma_kind(KIND, tbase, da + ao, db + bo, id, acc, 0, 0);
        } else if (BMODE == 1) {  // MN-major B only
          if (A_TMEM)
            mma_kind_ts(KIND, tbase, tbase + kTA + 8 * kk, db_mn + bo_mn, id_mn, acc);
          else
            mma_kind(KIND, tbase, da + ao, db_mn + bo_mn, id_mn, acc, 0, 0);
        } else {  // attention pattern: S-like group (K-major, smem A) then PV-like group (TMEM A, MN-major B)
          mma_kind(KIND, tbase + 256u * issuer, da + ao, db + bo, id, acc, 0, 0);
        }
      }
      if (BMODE == 2) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bo_mn = (uint64_t)((kk * ROWS_PER_MMA * 128) >> 4);
          const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
          if (SYNC & 8)  // two issuers: A from shared memory (no free TMEM columns for a second A)
            mma_kind(KIND, tbase + 256u * issuer + 128u, da + (uint64_t)(((kk >> 2) * 128 * 128 + (kk & 3) * 32) >> 4),
                     db_mn + bo_mn, id_mn, acc, 0, 0);
          else
            mma_kind_ts(KIND, tbase + 128, tbase + kTA + 8 * kk, db_mn + bo_mn, id_mn, acc);
        }
      }
      if (COMMIT) tc_commit(cb);
    }
    tc_commit(smem_u32(&bar[1 + 2 * issuer]));
    const bool ok = wait_bar(smem_u32(&bar[1 + 2 * issuer]), 0, abort_flag, 1000000000ull);
    tc_fence_after();
    const long long t1 = clock64();
    if (issuer == 0) {
      cycles[blockIdx.x] = (ok && seen) ? (unsigned long long)(t1 - t0) : (unsigned long long)(-5LL);
      *(reinterpret_cast<volatile int*>(abort_flag) + 1) = 1;  // stop the traffic warps
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <int ILP>
__global__ void ex2_loop_kernel(int iters, unsigned long long* cycles, float* sink) {
  float x[ILP];
#pragma unroll
  for (int u = 0; u < ILP; ++u) x[u] = 0.25f + 0.0625f * u + 1e-4f * (threadIdx.x & 31);
  __syncthreads();
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int u = 0; u < ILP; ++u) x[u] = ex2(-x[u]);  // stays in (1/2, 1)
  }
  __syncthreads();
  const long long t1 = clock64();
  float s = 0.f;
#pragma unroll
  for (int u = 0; u < ILP; ++u) s += x[u];
  sink[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
  if (threadIdx.x == 0) cycles[blockIdx.x] = (unsigned long long)(t1 - t0);
}

__global__ void softmax_loop_kernel(int iters, unsigned long long* cycles, float* sink) {
  uint64_t s[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) s[u] = f2(-0.5f - 0.03f * u, -0.25f - 0.01f * (threadIdx.x & 31));
  const uint64_t sc = f2(1.0f, 1.0f), negm = f2(0.0f, 0.0f);
  uint64_t lA = f2(0.f, 0.f), lB = f2(0.f, 0.f);
  uint32_t wacc = 0;
  __syncthreads();
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float x0, x1;
      f2_split(ffma2(s[u], sc, negm), x0, x1);
      const float p0 = ex2(x0), p1 = ex2(x1);
      if (u & 1) lB = fadd2(lB, f2(p0, p1));
      else lA = fadd2(lA, f2(p0, p1));
      wacc ^= pack_bf16(p0, p1);
      s[u] = f2(-p1, -p0);  // next step's scores: in (-1, -1/4], so 2^x stays in [1/2, 1)
    }
  }
  __syncthreads();
  const long long t1 = clock64();
  float a, b, c, d;
  f2_split(lA, a, b);
  f2_split(lB, c, d);
  sink[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = a + b + c + d + (float)(wacc & 0xFF);
  if (threadIdx.x == 0) cycles[blockIdx.x] = (unsigned long long)(t1 - t0);
}

}  // namespace tap

TAP_API int tap_mma_rate(int kind, int n, int iters, int grid, int flags, unsigned long long* cycles,
                         void* stream) {
  if (kind < TAP_KIND_BF16 || kind > TAP_KIND_F4 || iters < 1 || grid < 1 || !cycles) return -1;
  if (n != 128 && n != 256) return -1;
  if (kind == TAP_KIND_F4 && n != 128) return -1;
  if (flags & ~(TAP_A_TMEM | TAP_TWO_ACC | TAP_TWO_ISSUERS)) return -1;
  if ((flags & (TAP_TWO_ACC | TAP_TWO_ISSUERS)) && n != 128) return -1;
  if ((flags & TAP_TWO_ACC) && (flags & TAP_TWO_ISSUERS)) return -1;
  if ((flags & TAP_A_TMEM) && kind == TAP_KIND_F4) return -1;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(tap::mma_loop_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tap::kMmaSmem) !=
        cudaSuccess)
      return -4;
    attr_set = true;
  }
  tap::mma_loop_kernel<<<grid, 128, tap::kMmaSmem, reinterpret_cast<cudaStream_t>(stream)>>>(kind, n, iters,
                                                                                              flags, cycles);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

template <int KIND, int N, bool AT, bool CM, int BM = 0, int SY = 0>
static int launch_tight(int iters, int grid, unsigned long long* cycles, cudaStream_t st) {
  auto k = tap::mma_tight_kernel<KIND, N, AT, CM, BM, SY>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, tap::kMmaSmem) != cudaSuccess) return -4;
  k<<<grid, 128, tap::kMmaSmem, st>>>(iters, cycles);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

template <int KIND>
static int tight_dispatch(int n, int flags, int iters, int grid, unsigned long long* cycles, cudaStream_t st) {
  const bool at = flags & TAP_A_TMEM, cm = flags & TAP_COMMIT;
  if (flags & TAP_B_MN) {
    if (n != 128) return -1;
    return at ? launch_tight<KIND, 128, true, true, 1>(iters, grid, cycles, st)
              : launch_tight<KIND, 128, false, true, 1>(iters, grid, cycles, st);
  }
  if (flags & TAP_ATTN) {
    if (n != 128) return -1;
    const int sy = ((flags & TAP_TESTWAIT) ? 1 : 0) | ((flags & TAP_WAITFENCE) ? 2 : 0) |
                   ((flags & TAP_TMEM_TRAFFIC) ? 4 : 0) | ((flags & TAP_TWO_ISSUERS) ? 8 : 0) |
                   ((flags & TAP_FLAGPOLL) ? 16 : 0) | ((flags & TAP_FLAGFENCE) ? 32 : 0);
    switch (sy) {  // TMEM A initialised
      case 0: return launch_tight<KIND, 128, true, true, 2, 0>(iters, grid, cycles, st);
      case 1: return launch_tight<KIND, 128, true, true, 2, 1>(iters, grid, cycles, st);
      case 2: return launch_tight<KIND, 128, true, true, 2, 2>(iters, grid, cycles, st);
      case 3: return launch_tight<KIND, 128, true, true, 2, 3>(iters, grid, cycles, st);
      case 4: return launch_tight<KIND, 128, true, true, 2, 4>(iters, grid, cycles, st);
      case 7: return launch_tight<KIND, 128, true, true, 2, 7>(iters, grid, cycles, st);
      case 8: return launch_tight<KIND, 128, true, true, 2, 8>(iters, grid, cycles, st);
      case 11: return launch_tight<KIND, 128, true, true, 2, 11>(iters, grid, cycles, st);
      case 16: return launch_tight<KIND, 128, true, true, 2, 16>(iters, grid, cycles, st);
      case 32: return launch_tight<KIND, 128, true, true, 2, 32>(iters, grid, cycles, st);
      case 48: return launch_tight<KIND, 128, true, true, 2, 48>(iters, grid, cycles, st);
      default: return -1;
    }
  }
  if (flags & (TAP_TESTWAIT | TAP_WAITFENCE | TAP_TMEM_TRAFFIC | TAP_FLAGPOLL | TAP_FLAGFENCE)) return -1;
  if (n == 128) {
    if (at) return cm ? launch_tight<KIND, 128, true, true>(iters, grid, cycles, st)
                      : launch_tight<KIND, 128, true, false>(iters, grid, cycles, st);
    return cm ? launch_tight<KIND, 128, false, true>(iters, grid, cycles, st)
              : launch_tight<KIND, 128, false, false>(iters, grid, cycles, st);
  }
  if (at) return cm ? launch_tight<KIND, 256, true, true>(iters, grid, cycles, st)
                    : launch_tight<KIND, 256, true, false>(iters, grid, cycles, st);
  return cm ? launch_tight<KIND, 256, false, true>(iters, grid, cycles, st)
            : launch_tight<KIND, 256, false, false>(iters, grid, cycles, st);
}

TAP_API int tap_mma_tight_rate(int kind, int n, int iters, int grid, int flags, unsigned long long* cycles,
                               void* stream) {
  if (iters < 1 || grid < 1 || !cycles || (n != 128 && n != 256)) return -1;
  if (flags & ~(TAP_A_TMEM | TAP_COMMIT | TAP_B_MN | TAP_ATTN | TAP_TESTWAIT | TAP_WAITFENCE | TAP_TMEM_TRAFFIC |
                TAP_TWO_ISSUERS | TAP_FLAGPOLL | TAP_FLAGFENCE))
    return -1;
  if ((flags & TAP_TWO_ISSUERS) && !(flags & TAP_ATTN)) return -1;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (kind) {
    case TAP_KIND_BF16: return tight_dispatch<TAP_KIND_BF16>(n, flags, iters, grid, cycles, st);
    case TAP_KIND_I8: return tight_dispatch<TAP_KIND_I8>(n, flags, iters, grid, cycles, st);
    case TAP_KIND_F8: return tight_dispatch<TAP_KIND_F8>(n, flags, iters, grid, cycles, st);
    case TAP_KIND_F4:
      if (n != 128 || flags & ~TAP_COMMIT) return -1;
      return (flags & TAP_COMMIT) ? launch_tight<TAP_KIND_F4, 128, false, true>(iters, grid, cycles, st)
                                  : launch_tight<TAP_KIND_F4, 128, false, false>(iters, grid, cycles, st);
    default: return -1;
  }
}

TAP_API int tap_ex2_rate(int threads, int ilp, int iters, int grid, unsigned long long* cycles, float* sink,
                         void* stream) {
  if (threads < 32 || threads > 1024 || threads % 32 || iters < 1 || grid < 1 || !cycles || !sink) return -1;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (ilp) {
    case 1: tap::ex2_loop_kernel<1><<<grid, threads, 0, st>>>(iters, cycles, sink); break;
    case 2: tap::ex2_loop_kernel<2><<<grid, threads, 0, st>>>(iters, cycles, sink); break;
    case 4: tap::ex2_loop_kernel<4><<<grid, threads, 0, st>>>(iters, cycles, sink); break;
    case 8: tap::ex2_loop_kernel<8><<<grid, threads, 0, st>>>(iters, cycles, sink); break;
    default: return -1;
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

TAP_API int tap_softmax_rate(int threads, int iters, int grid, unsigned long long* cycles, float* sink,
                             void* stream) {
  if (threads < 32 || threads > 1024 || threads % 32 || iters < 1 || grid < 1 || !cycles || !sink) return -1;
  tap::softmax_loop_kernel<<<grid, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(iters, cycles, sink);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}
