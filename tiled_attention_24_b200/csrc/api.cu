// C-ABI entry points of libtiledattn (declared in include/tiledattn.h):
// argument validation, TMA descriptor construction, launches.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "tiledattn.h"
#include "ptx.cuh"
#include "fwd_bf16.cuh"
#include "decode.cuh"
#include "quant.cuh"
#include "fwd_int8.cuh"
#include "fwd_fp4.cuh"
#include "bwd_bf16.cuh"
#include "fwd_fp8.cuh"
#include "decode_tc.cuh"

namespace {

constexpr unsigned long long kDefaultWaitNs = 1000000000ull;
unsigned long long g_wait_ns = kDefaultWaitNs;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [BH][N][d] bf16 viewed as a 3-D tensor (d, N, BH); boxes of 64 x box_rows
// x 1 with 128-byte swizzle.  Rows past N read as zero and are not written.
int make_tmap_bf16(CUtensorMap* m, const void* ptr, int d, int N, int BH, int box_rows = 128) {
  auto enc = encode_fn();
  if (!enc) return ATTN_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// [rows][d] bf16 viewed as a 2-D tensor (d, rows); boxes of 64 x box_rows with
// 128-byte swizzle.  Rows past `rows` read as zero.
int make_tmap_rows(CUtensorMap* m, const void* ptr, int d, long long rows, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return ATTN_ERR_CUDA;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// Packed token-major bf16 [total][heads][d] viewed as (d, heads, total);
// boxes of 64 x 1 x 128 (the same 128-row x 128-byte smem tile as
// make_tmap_bf16's boxes) with 128-byte swizzle.  Rows past total read as zero.
int make_tmap_tok(CUtensorMap* m, const void* ptr, int d, int heads, int total) {
  auto enc = encode_fn();
  if (!enc) return ATTN_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)total};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// [BH][N][128] int8 viewed as (128, N, BH); boxes of 128 x 128 x 1 bytes with
// 128-byte swizzle.
int make_tmap_i8(CUtensorMap* m, const void* ptr, int N, int BH) {
  auto enc = encode_fn();
  if (!enc) return ATTN_ERR_CUDA;
  cuuint64_t dims[3] = {128, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {128, (cuuint64_t)N * 128};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// packed e2m1 codes viewed as (row_bytes, rows, BH) bytes; boxes of 64 x 128 x 1
// with 64-byte swizzle (one swizzle span per 128-code row)
int make_tmap_fp4(CUtensorMap* m, const void* ptr, long long row_bytes, int rows, int BH) {
  auto enc = encode_fn();
  if (!enc) return ATTN_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)row_bytes, (cuuint64_t)rows, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)row_bytes * rows};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

template <bool SCORES_ONLY>
int launch_fp4(const void* q, const void* qsf, const void* k, const void* ksf, const void* vt, const void* vsf,
               float* o, float* lse, float* s_out, int B, int H, int Nq, int Nkv, int causal, float scale,
               int p_mode, cudaStream_t st) {
  using C = ta::FwdF4Cfg;
  const int BH = B * H;
  const int KT = (Nkv + 127) / 128;
  CUtensorMap tq, tk, tv;
  int rc;
  if ((rc = make_tmap_fp4(&tq, q, 64, Nq, BH)) != ATTN_OK) return rc;
  if ((rc = make_tmap_fp4(&tk, k, 64, Nkv, BH)) != ATTN_OK) return rc;
  if ((rc = make_tmap_fp4(&tv, SCORES_ONLY ? k : vt, SCORES_ONLY ? 64 : (long long)KT * 64,
                          SCORES_ONLY ? Nkv : 128, BH)) != ATTN_OK)
    return rc;
  if (cudaFuncSetAttribute(ta::fwd_fp4_kernel<SCORES_ONLY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM) != cudaSuccess)
    return ATTN_ERR_CUDA;
  ta::FwdF4Params p;
  p.q_sf = static_cast<const uint8_t*>(qsf);
  p.k_sf = static_cast<const uint8_t*>(ksf);
  p.v_sf = static_cast<const uint8_t*>(vsf);
  p.o = o;
  p.lse = lse;
  p.s_out = s_out;
  p.Nq = Nq;
  p.Nkv = Nkv;
  p.n_qp = (Nq + 255) / 256;
  p.Tc = KT;
  p.RTq = (Nq + 127) / 128;
  p.KT = KT;
  p.causal = causal ? 1 : 0;
  p.p_mode = p_mode;
  p.sl2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_wait_ns;
  const long long grid = (long long)BH * p.n_qp;
  if (grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  ta::fwd_fp4_kernel<SCORES_ONLY><<<(unsigned)grid, C::THREADS, C::SMEM, st>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <bool SCORES_ONLY>
int launch_int8(const void* q, const float* qs, const void* k, const float* ks, const void* v, const float* vs,
                float* o, float* lse, int* s_out, int B, int H, int Nq, int Nkv, int causal, float scale,
                cudaStream_t st) {
  using C = ta::FwdI8Cfg;
  const int BH = B * H;
  CUtensorMap tq, tk, tv;
  int rc;
  if ((rc = make_tmap_i8(&tq, q, Nq, BH)) != ATTN_OK) return rc;
  if ((rc = make_tmap_i8(&tk, k, Nkv, BH)) != ATTN_OK) return rc;
  if ((rc = make_tmap_i8(&tv, SCORES_ONLY ? k : v, Nkv, BH)) != ATTN_OK) return rc;
  if (cudaFuncSetAttribute(ta::fwd_int8_kernel<SCORES_ONLY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM) != cudaSuccess)
    return ATTN_ERR_CUDA;
  ta::FwdI8Params p;
  p.q_scale = qs;
  p.k_scale = ks;
  p.v_scale = vs;
  p.o = o;
  p.lse = lse;
  p.s_out = s_out;
  p.Nq = Nq;
  p.Nkv = Nkv;
  p.n_qt = (Nq + 127) / 128;
  p.Tc = (Nkv + 127) / 128;
  p.causal = causal ? 1 : 0;
  p.ks_vec = (ks != nullptr) && (Nkv % 4 == 0) && aligned16(ks);
  p.sl2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_wait_ns;
  const long long grid = (long long)BH * p.n_qt;
  if (grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  ta::fwd_int8_kernel<SCORES_ONLY><<<(unsigned)grid, C::THREADS, C::SMEM, st>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <typename K>
int set_smem_attr(K kernel, int bytes) {
  // cheap, idempotent; done per call so that every device the caller uses is covered
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
             ? ATTN_OK
             : ATTN_ERR_CUDA;
}

template <int D>
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv, int Nq,
               int Nkv, int causal, float scale, cudaStream_t st) {
  using C = ta::FwdCfg<D>;
  const int BH = B * H;
  CUtensorMap tq, tk, tv, to;
  int rc;
  if ((rc = make_tmap_bf16(&tq, q, D, Nq, BH)) != ATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&tk, k, D, Nkv, B * Hkv)) != ATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&tv, v, D, Nkv, B * Hkv)) != ATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&to, o, D, Nq, BH)) != ATTN_OK) return rc;
  if ((rc = set_smem_attr(ta::fwd_bf16_kernel<D>, C::SMEM)) != ATTN_OK) return rc;
  ta::FwdParams p{};
  p.lse = lse;
  p.Nq = Nq;
  p.Nkv = Nkv;
  p.n_qp = (Nq + 255) / 256;
  p.Tc = (Nkv + 127) / 128;
  p.group = H / Hkv;
  p.causal = causal ? 1 : 0;
  p.sl2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_wait_ns;
  {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    p.wave = sms;  // one CTA per SM (shared memory)
  }
  const long long grid = (long long)BH * p.n_qp;
  if (grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  ta::fwd_bf16_kernel<D><<<(unsigned)grid, C::THREADS, C::SMEM, st>>>(tq, tk, tv, to, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D>
int launch_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_q,
                      const int* cu_k, int B, int H, int Hkv, int total_q, int total_k, int max_q, int causal,
                      float scale, cudaStream_t st) {
  using C = ta::FwdCfg<D>;
  CUtensorMap tq, tk, tv;
  int rc;
  if ((rc = make_tmap_tok(&tq, q, D, H, total_q)) != ATTN_OK) return rc;
  if ((rc = make_tmap_tok(&tk, k, D, Hkv, total_k)) != ATTN_OK) return rc;
  if ((rc = make_tmap_tok(&tv, v, D, Hkv, total_k)) != ATTN_OK) return rc;
  if ((rc = set_smem_attr(ta::fwd_bf16_kernel<D, true>, C::SMEM)) != ATTN_OK) return rc;
  ta::FwdParams p{};
  p.lse = lse;
  p.Nq = 0;
  p.Nkv = 0;
  p.n_qp = (max_q + 255) / 256;
  p.Tc = 0;
  p.group = H / Hkv;
  p.causal = causal ? 1 : 0;
  p.sl2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_wait_ns;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.o = static_cast<uint16_t*>(o);
  p.nb = B;
  p.H = H;
  p.total_q = total_q;
  p.total_k = total_k;
  const long long grid = (long long)B * H * p.n_qp;
  if (grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  // tmO is not used by the variable-length epilogue (direct stores); any valid map will do
  ta::fwd_bf16_kernel<D, true><<<(unsigned)grid, C::THREADS, C::SMEM, st>>>(tq, tk, tv, tq, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool P8>
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
               void* dq, void* dk, void* dv, float* rowdot, int B, int H, int Nq, int Nkv, int causal, float scale,
               cudaStream_t st) {
  using C = ta::BwdCfg<D>;
  const int BH = B * H;
  CUtensorMap tq, tk, tv, tdo;
  int rc;
  if ((rc = make_tmap_bf16(&tq, q, D, Nq, BH)) != ATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&tk, k, D, Nkv, BH)) != ATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&tv, v, D, Nkv, BH)) != ATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&tdo, dout, D, Nq, BH)) != ATTN_OK) return rc;
  if ((rc = set_smem_attr(ta::bwd_dkdv_kernel<D, P8>, C::SMEM)) != ATTN_OK) return rc;
  if ((rc = set_smem_attr(ta::bwd_dq_kernel<D>, C::SMEM)) != ATTN_OK) return rc;
  ta::BwdParams p;
  p.o = static_cast<const uint16_t*>(o);
  p.dout = static_cast<const uint16_t*>(dout);
  p.lse = lse;
  p.rowdot = rowdot;
  p.dq = static_cast<uint16_t*>(dq);
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  p.Nq = Nq;
  p.Nkv = Nkv;
  p.nqt = (Nq + 127) / 128;
  p.nkt = (Nkv + 127) / 128;
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.sl2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_wait_ns;
  const long long rows = (long long)BH * Nq;
  const long long gk = (long long)BH * p.nkt, gq = (long long)BH * p.nqt;
  if ((rows + 7) / 8 > 0x7fffffffLL || gk > 0x7fffffffLL || gq > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  ta::bwd_rowdot_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(p.o, p.dout, rowdot, rows);
  ta::bwd_dkdv_kernel<D, P8><<<(unsigned)gk, C::THREADS, C::SMEM, st>>>(tq, tk, tv, tdo, p);
  ta::bwd_dq_kernel<D><<<(unsigned)gq, C::THREADS, C::SMEM, st>>>(tq, tk, tv, tdo, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

size_t decode_ws_bytes(long long BH, int d, int S) {
  const size_t o_bytes = (size_t)BH * S * d * sizeof(float);
  const size_t l_bytes = (size_t)BH * S * sizeof(float);
  return ((o_bytes + 255) & ~size_t(255)) + l_bytes;
}

// Fixed scratch for attn_decode_noalloc: split partials (O then LSE), shared
// by every call of that entry point on a device.
static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[ATTN_DECODE_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array per device, looked up once per device
// with cudaGetSymbolAddress (in host code the array's name is only a stand-in).
constexpr int kMaxDevices = 64;
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

int noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_noalloc_scratch) != cudaSuccess || !p) return ATTN_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return ATTN_OK;
}

__global__ void watchdog_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ta::mbar_init(ta::smem_u32(&bar), 1);
    abort_flag = 0;
    ta::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives: the bounded wait must give up and record a timeout
    ta::wait_bar(ta::smem_u32(&bar), 0, &abort_flag, limit_ns);
  }
  __syncthreads();
}

}  // namespace

template <int G>
static int launch_decode_tc_g(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, float* o_part,
                              float* l_part, long long BH, int Nkv, int S, int chunk, float sl2, int grp,
                              const int* seqlens, int H, cudaStream_t st) {
  using C = ta::DecTcCfg;
  if (cudaFuncSetAttribute(ta::decode_gqa_tc_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
      cudaSuccess)
    return ATTN_ERR_CUDA;
  const long long items = BH / G * S;
  if (items > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  // persistent: two CTAs per SM, each walking items with a stride of the grid
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return ATTN_ERR_CUDA;
  const unsigned grid = (unsigned)std::min<long long>(items, 2LL * sms);
  ta::decode_gqa_tc_kernel<G><<<grid, C::THREADS, C::SMEM, st>>>(tq, tk, tv, o_part, l_part, (int)items, Nkv, S,
                                                                  chunk, sl2, grp, seqlens, H, g_wait_ns);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Grouped-query decode on the tensor cores (d = 128): G query heads per CTA.
static int launch_decode_tc(const void* q, const void* k, const void* v, float* o_part, float* l_part, int B, int H,
                            int Hkv, int Nkv, int G, int S, int chunk, float sl2, int grp, const int* seqlens,
                            cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  int rc;
  if ((rc = make_tmap_rows(&tq, q, 128, (long long)B * H, 8)) != ATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&tk, k, 128, Nkv, B * Hkv, ta::DecTcCfg::KT)) != ATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&tv, v, 128, Nkv, B * Hkv, ta::DecTcCfg::KT)) != ATTN_OK) return rc;
  const long long BH = (long long)B * H;
  switch (G) {
    case 8: return launch_decode_tc_g<8>(tq, tk, tv, o_part, l_part, BH, Nkv, S, chunk, sl2, grp, seqlens, H, st);
    case 7: return launch_decode_tc_g<7>(tq, tk, tv, o_part, l_part, BH, Nkv, S, chunk, sl2, grp, seqlens, H, st);
    case 6: return launch_decode_tc_g<6>(tq, tk, tv, o_part, l_part, BH, Nkv, S, chunk, sl2, grp, seqlens, H, st);
    case 5: return launch_decode_tc_g<5>(tq, tk, tv, o_part, l_part, BH, Nkv, S, chunk, sl2, grp, seqlens, H, st);
    case 4: return launch_decode_tc_g<4>(tq, tk, tv, o_part, l_part, BH, Nkv, S, chunk, sl2, grp, seqlens, H, st);
    case 3: return launch_decode_tc_g<3>(tq, tk, tv, o_part, l_part, BH, Nkv, S, chunk, sl2, grp, seqlens, H, st);
    case 2: return launch_decode_tc_g<2>(tq, tk, tv, o_part, l_part, BH, Nkv, S, chunk, sl2, grp, seqlens, H, st);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

extern "C" {

const char* attn_status_string(int s) {
  switch (s) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_MISALIGNED: return "ATTN_ERR_MISALIGNED";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    case ATTN_ERR_TOO_LARGE: return "ATTN_ERR_TOO_LARGE";
    case ATTN_ERR_BOUNDS: return "ATTN_ERR_BOUNDS";
    default: return "ATTN_ERR_UNKNOWN";
  }
}

const char* attn_version(void) { return "tiledattn 0.1 sm_100a"; }

void attn_set_wait_limit_ns(unsigned long long ns) { g_wait_ns = ns ? ns : kDefaultWaitNs; }

int attn_fwd_gqa(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o, float* lse,
                 int B, int H, int Hkv, int Nq, int Nkv, int d, int causal, float scale, void* stream) {
  if (B < 0 || H < 0 || Nq < 0 || Nkv < 0) return ATTN_ERR_INVALID_ARG;
  if (Hkv < 1 || (H > 0 && H % Hkv != 0) || Hkv > (H > 0 ? H : Hkv)) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * H > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || Nq == 0) return ATTN_OK;
  if (!q || !o || !lse || (Nkv > 0 && (!k || !v))) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned4(lse) || (Nkv > 0 && (!aligned16(k) || !aligned16(v))))
    return ATTN_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (Nkv == 0) {
    const long long rows = (long long)B * H * Nq;
    const long long n = rows * d;
    const long long blocks = (n + 255) / 256;
    if (blocks > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    ta::fill_empty_kernel<<<(unsigned)blocks, 256, 0, st>>>(o, lse, rows, d);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  return d == 128 ? launch_fwd<128>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, causal, scale, st)
                  : launch_fwd<64>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, causal, scale, st);
}

int attn_fwd_varlen(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o, float* lse,
                    const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H, int Hkv, int total_q,
                    int total_k, int max_seqlen_q, int d, int causal, float scale, void* stream) {
  if (B < 0 || H < 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0) return ATTN_ERR_INVALID_ARG;
  if (Hkv < 1 || (H > 0 && H % Hkv != 0) || Hkv > (H > 0 ? H : Hkv)) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || total_q == 0) return ATTN_OK;
  if (!q || !o || !lse || !cu_seqlens_q || !cu_seqlens_k || (total_k > 0 && (!k || !v))) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned4(lse) || !aligned4(cu_seqlens_q) || !aligned4(cu_seqlens_k) ||
      (total_k > 0 && (!aligned16(k) || !aligned16(v))))
    return ATTN_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (total_k == 0) {  // no keys anywhere: every row gets O = 0, LSE = -inf
    const long long rows = (long long)total_q * H;
    const long long blocks = (rows * d + 255) / 256;
    if (blocks > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    ta::fill_empty_kernel<<<(unsigned)blocks, 256, 0, st>>>(o, lse, rows, d);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  if (max_seqlen_q == 0) return ATTN_OK;
  return d == 128 ? launch_fwd_varlen<128>(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, H, Hkv, total_q, total_k,
                                           max_seqlen_q, causal, scale, st)
                  : launch_fwd_varlen<64>(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, H, Hkv, total_q, total_k,
                                          max_seqlen_q, causal, scale, st);
}

int attn_fwd(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o, float* lse,
             int B, int H, int Nq, int Nkv, int d, int causal, float scale, void* stream) {
  return attn_fwd_gqa(q, k, v, o, lse, B, H, H > 0 ? H : 1, Nq, Nkv, d, causal, scale, stream);
}

size_t attn_bwd_workspace_bytes(int B, int H, int Nq) {
  if (B <= 0 || H <= 0 || Nq <= 0) return 0;
  return ((size_t)B * H * Nq * sizeof(float) + 255) & ~size_t(255);
}

static int bwd_impl(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, const attn_bf16_t* o,
                    const attn_bf16_t* dout, const float* lse, attn_bf16_t* dq, attn_bf16_t* dk, attn_bf16_t* dv,
                    int B, int H, int Nq, int Nkv, int d, int causal, float scale, void* workspace,
                    size_t workspace_bytes, void* stream, bool p8) {
  if (B < 0 || H < 0 || Nq < 0 || Nkv < 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * H > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0) return ATTN_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t kv_bytes = (size_t)B * H * Nkv * d * 2, q_bytes = (size_t)B * H * Nq * d * 2;
  if (Nq == 0 || Nkv == 0) {
    // no query or no key: every gradient that exists is zero
    if (Nkv > 0 && (!dk || !dv)) return ATTN_ERR_INVALID_ARG;
    if (Nq > 0 && !dq) return ATTN_ERR_INVALID_ARG;
    if (Nkv > 0 && (cudaMemsetAsync(dk, 0, kv_bytes, st) != cudaSuccess ||
                    cudaMemsetAsync(dv, 0, kv_bytes, st) != cudaSuccess))
      return ATTN_ERR_CUDA;
    if (Nq > 0 && cudaMemsetAsync(dq, 0, q_bytes, st) != cudaSuccess) return ATTN_ERR_CUDA;
    return ATTN_OK;
  }
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned4(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
    return ATTN_ERR_MISALIGNED;
  if (workspace_bytes < attn_bwd_workspace_bytes(B, H, Nq)) return ATTN_ERR_INVALID_ARG;
  float* rowdot = static_cast<float*>(workspace);
  if (p8)
    return d == 128 ? launch_bwd<128, true>(q, k, v, o, dout, lse, dq, dk, dv, rowdot, B, H, Nq, Nkv, causal, scale, st)
                    : launch_bwd<64, true>(q, k, v, o, dout, lse, dq, dk, dv, rowdot, B, H, Nq, Nkv, causal, scale, st);
  return d == 128 ? launch_bwd<128, false>(q, k, v, o, dout, lse, dq, dk, dv, rowdot, B, H, Nq, Nkv, causal, scale, st)
                  : launch_bwd<64, false>(q, k, v, o, dout, lse, dq, dk, dv, rowdot, B, H, Nq, Nkv, causal, scale, st);
}

int attn_bwd(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, const attn_bf16_t* o,
             const attn_bf16_t* dout, const float* lse, attn_bf16_t* dq, attn_bf16_t* dk, attn_bf16_t* dv, int B,
             int H, int Nq, int Nkv, int d, int causal, float scale, void* workspace, size_t workspace_bytes,
             void* stream) {
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, Nq, Nkv, d, causal, scale, workspace, workspace_bytes,
                  stream, false);
}

int attn_bwd_fp8p(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, const attn_bf16_t* o,
                  const attn_bf16_t* dout, const float* lse, attn_bf16_t* dq, attn_bf16_t* dk, attn_bf16_t* dv,
                  int B, int H, int Nq, int Nkv, int d, int causal, float scale, void* workspace,
                  size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, Nq, Nkv, d, causal, scale, workspace, workspace_bytes,
                  stream, true);
}

size_t attn_decode_workspace_bytes(int B, int H, int d, int num_splits) {
  if (B <= 0 || H <= 0 || num_splits <= 0 || (d != 64 && d != 128)) return 0;
  return decode_ws_bytes((long long)B * H, d, num_splits);
}

static int decode_impl(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o,
                       float* lse, const int* seqlens, int B, int H, int Hkv, int Nkv, int d, float scale,
                       int num_splits, void* workspace, size_t workspace_bytes, void* stream) {
  if (B < 0 || H < 0 || Nkv < 1) return ATTN_ERR_INVALID_ARG;
  if (Hkv < 1 || (H > 0 && H % Hkv != 0) || Hkv > (H > 0 ? H : Hkv)) return ATTN_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > 1024) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0) return ATTN_OK;
  const long long BH = (long long)B * H;
  if (BH * num_splits > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o || !lse || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(lse) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(o) & 1u))
    return ATTN_ERR_MISALIGNED;
  if (workspace_bytes < decode_ws_bytes(BH, d, num_splits)) return ATTN_ERR_INVALID_ARG;
  const int chunk = (int)((Nkv + (long long)num_splits - 1) / num_splits);
  float* o_part = static_cast<float*>(workspace);
  float* l_part = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                           (((size_t)BH * num_splits * d * sizeof(float) + 255) & ~size_t(255)));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float sl2 = scale * 1.4426950408889634f;
  // query heads per CTA: the largest of 4, 2 dividing the group (each cache
  // row then crosses memory once per G query heads; a group of 8 runs as two
  // CTAs of 4, the second reading the cache head from L2); 1 = plain kernel.
  // Eight heads in one CTA take 255 registers and two CTAs per SM, too few
  // loads in flight: 1560 GB/s against 2260 as two CTAs of 4 (B64 Hq32
  // Hkv4 N_kv 8192 d128).
  const int grp = H / Hkv;
  if (d == 128 && grp > 1) {
    // tensor-core kernel: up to 8 query heads of a group per CTA (the largest
    // divisor of the group that is <= 8)
    int G = 8;
    while (grp % G) --G;
    int rc = launch_decode_tc(q, k, v, o_part, l_part, B, H, Hkv, Nkv, G, num_splits, chunk, sl2, grp, seqlens, st);
    if (rc != ATTN_OK) return rc;
    ta::decode_combine_kernel<128><<<(unsigned)BH, 128, 0, st>>>(o_part, l_part, o, lse, num_splits);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  const int G = (grp % 4 == 0) ? 4 : (grp % 2 == 0) ? 2 : 1;
  const unsigned grid = (unsigned)(BH / G * num_splits);
  if (G == 1) {
    if (d == 128)
      ta::decode_split_kernel<128><<<grid, ta::DEC_THREADS, 0, st>>>(q, k, v, o_part, l_part, Nkv, num_splits, chunk,
                                                                      sl2, grp, seqlens, H);
    else
      ta::decode_split_kernel<64><<<grid, ta::DEC_THREADS, 0, st>>>(q, k, v, o_part, l_part, Nkv, num_splits, chunk,
                                                                     sl2, grp, seqlens, H);
  } else {
#define TA_DECODE_GROUP(DD, GG)                                                                           \
  ta::decode_split_group_kernel<DD, GG><<<grid, ta::DEC_THREADS, 0, st>>>(q, k, v, o_part, l_part, Nkv, \
                                                                         num_splits, chunk, sl2, grp, seqlens, H)
    if (d == 128) {
      if (G == 4) TA_DECODE_GROUP(128, 4); else TA_DECODE_GROUP(128, 2);
    } else {
      if (G == 4) TA_DECODE_GROUP(64, 4); else TA_DECODE_GROUP(64, 2);
    }
#undef TA_DECODE_GROUP
  }
  if (d == 128)
    ta::decode_combine_kernel<128><<<(unsigned)BH, 128, 0, st>>>(o_part, l_part, o, lse, num_splits);
  else
    ta::decode_combine_kernel<64><<<(unsigned)BH, 64, 0, st>>>(o_part, l_part, o, lse, num_splits);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_decode_gqa(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o,
                    float* lse, int B, int H, int Hkv, int Nkv, int d, float scale, int num_splits,
                    void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(q, k, v, o, lse, nullptr, B, H, Hkv, Nkv, d, scale, num_splits, workspace, workspace_bytes,
                     stream);
}

int attn_decode_varlen(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o,
                       float* lse, const int* seqlens_k, int B, int H, int Hkv, int Nkv_max, int d, float scale,
                       int num_splits, void* workspace, size_t workspace_bytes, void* stream) {
  if (B > 0 && H > 0 && !seqlens_k) return ATTN_ERR_INVALID_ARG;
  if (seqlens_k && !aligned4(seqlens_k)) return ATTN_ERR_MISALIGNED;
  return decode_impl(q, k, v, o, lse, seqlens_k, B, H, Hkv, Nkv_max, d, scale, num_splits, workspace,
                     workspace_bytes, stream);
}

int attn_decode(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o, float* lse,
                int B, int H, int Nkv, int d, float scale, int num_splits, void* workspace,
                size_t workspace_bytes, void* stream) {
  return attn_decode_gqa(q, k, v, o, lse, B, H, H > 0 ? H : 1, Nkv, d, scale, num_splits, workspace,
                         workspace_bytes, stream);
}

int attn_decode_noalloc(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o,
                        float* lse, int B, int H, int Nkv, int d, float scale, int num_splits, void* stream) {
  if (B < 0 || H < 0 || Nkv < 1) return ATTN_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > 1024) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0) return ATTN_OK;
  const long long BH = (long long)B * H;
  if (BH * num_splits > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (decode_ws_bytes(BH, d, num_splits) > (size_t)ATTN_DECODE_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_TOO_LARGE;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(lse) || (reinterpret_cast<uintptr_t>(o) & 1u))
    return ATTN_ERR_MISALIGNED;
  void* scratch = nullptr;
  const int rc = noalloc_scratch(&scratch);
  if (rc != ATTN_OK) return rc;
  const int chunk = (int)((Nkv + (long long)num_splits - 1) / num_splits);
  float* o_part = static_cast<float*>(scratch);
  float* l_part = reinterpret_cast<float*>(static_cast<char*>(scratch) +
                                           (((size_t)BH * num_splits * d * sizeof(float) + 255) & ~size_t(255)));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float sl2 = scale * 1.4426950408889634f;
  const unsigned grid = (unsigned)(BH * num_splits);
  if (d == 128) {
    ta::decode_split_kernel<128><<<grid, ta::DEC_THREADS, 0, st>>>(q, k, v, o_part, l_part, Nkv, num_splits,
                                                                    chunk, sl2, 1, nullptr, H);
    ta::decode_combine_kernel<128><<<(unsigned)BH, 128, 0, st>>>(o_part, l_part, o, lse, num_splits);
  } else {
    ta::decode_split_kernel<64><<<grid, ta::DEC_THREADS, 0, st>>>(q, k, v, o_part, l_part, Nkv, num_splits,
                                                                   chunk, sl2, 1, nullptr, H);
    ta::decode_combine_kernel<64><<<(unsigned)BH, 64, 0, st>>>(o_part, l_part, o, lse, num_splits);
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_quantize_int8(const attn_bf16_t* x, int8_t* xq, float* xs, int B, int H, int N, int d, int per_head,
                       void* stream) {
  if (B < 0 || H < 0 || N < 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || N == 0) return ATTN_OK;
  if (!x || !xq || !xs) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xq) || !aligned4(xs)) return ATTN_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const long long BH = (long long)B * H;
  if (!per_head) {
    const long long rows = BH * N;
    const long long per_block = (d == 128) ? ta::qrow_rows_per_block<128>() : ta::qrow_rows_per_block<64>();
    const long long blocks = (rows + per_block - 1) / per_block;
    if (blocks > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    if (d == 128)
      ta::quant_int8_rows_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(x, xq, xs, rows);
    else
      ta::quant_int8_rows_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(x, xq, xs, rows);
  } else {
    if (BH > 65535) return ATTN_ERR_UNSUPPORTED;
    const long long per_head_n = (long long)N * d;  // multiple of 8 (d is)
    unsigned* amax = reinterpret_cast<unsigned*>(xs);
    if (cudaMemsetAsync(amax, 0, BH * sizeof(float), st) != cudaSuccess) return ATTN_ERR_CUDA;
    const unsigned gx = (unsigned)std::min<long long>(64, (per_head_n + 2047) / 2048);
    ta::head_amax_kernel<<<dim3(gx, (unsigned)BH), 256, 0, st>>>(x, amax, per_head_n);
    ta::quant_int8_heads_kernel<<<dim3(gx, (unsigned)BH), 256, 0, st>>>(x, xq, amax, per_head_n);
    ta::head_scale_kernel<<<(unsigned)((BH + 255) / 256), 256, 0, st>>>(amax, (int)BH);
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_quantize_int4(const attn_bf16_t* x, int8_t* xq, float* xs, int B, int H, int N, int d, void* stream) {
  if (B < 0 || H < 0 || N < 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || N == 0) return ATTN_OK;
  if (!x || !xq || !xs) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xq) || !aligned4(xs)) return ATTN_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const long long rows = (long long)B * H * N;
  const long long per_block = (d == 128) ? ta::qrow_rows_per_block<128>() : ta::qrow_rows_per_block<64>();
  const long long blocks = (rows + per_block - 1) / per_block;
  if (blocks > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (d == 128)
    ta::quant_int8_rows_kernel<128, 7><<<(unsigned)blocks, 256, 0, st>>>(x, xq, xs, rows);
  else
    ta::quant_int8_rows_kernel<64, 7><<<(unsigned)blocks, 256, 0, st>>>(x, xq, xs, rows);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_fwd_int8(const int8_t* q, const float* q_scale, const int8_t* k, const float* k_scale, const int8_t* v,
                  const float* v_scale, float* o, float* lse, int B, int H, int Nq, int Nkv, int d, int causal,
                  float scale, void* stream) {
  if (B < 0 || H < 0 || Nq < 0 || Nkv < 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * H > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || Nq == 0) return ATTN_OK;
  if (Nkv == 0) return ATTN_ERR_UNSUPPORTED;
  if (!q || !q_scale || !k || !k_scale || !v || !v_scale || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(q_scale) ||
      !aligned4(k_scale) || !aligned4(v_scale) || !aligned4(lse))
    return ATTN_ERR_MISALIGNED;
  return launch_int8<false>(q, q_scale, k, k_scale, v, v_scale, o, lse, nullptr, B, H, Nq, Nkv, causal, scale,
                            reinterpret_cast<cudaStream_t>(stream));
}

int attn_int8_scores(const int8_t* q, const int8_t* k, int32_t* s, int B, int H, int Nq, int Nkv, int d,
                     void* stream) {
  if (B < 0 || H < 0 || Nq < 0 || Nkv < 0) return ATTN_ERR_INVALID_ARG;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || Nq == 0 || Nkv == 0) return ATTN_OK;
  if (!q || !k || !s) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned4(s)) return ATTN_ERR_MISALIGNED;
  return launch_int8<true>(q, nullptr, k, nullptr, nullptr, nullptr, nullptr, nullptr, s, B, H, Nq, Nkv, 0, 1.f,
                           reinterpret_cast<cudaStream_t>(stream));
}

int attn_quantize_fp8(const attn_bf16_t* x, uint8_t* codes, float* scales, int B, int H, int N, int d, int mode,
                      const float* signs, void* stream) {
  if (B < 0 || H < 0 || N < 0 || (mode != 0 && mode != 1)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (mode == 1 && signs != nullptr) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0) return ATTN_OK;
  if (!x || !codes || !scales) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned4(scales) || (signs && !aligned4(signs)))
    return ATTN_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const long long BH = (long long)B * H;
  if (mode == 0) {
    const long long rows = BH * N;
    const long long per_block = (d == 128) ? ta::qrow_rows_per_block<128>() : ta::qrow_rows_per_block<64>();
    const long long blocks = (rows + per_block - 1) / per_block;
    if (blocks > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    if (d == 128)
      ta::quant_fp8_rows_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(x, signs, codes, scales, rows);
    else
      ta::quant_fp8_rows_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(x, signs, codes, scales, rows);
  } else {
    if (BH > 65535 || BH * d > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    unsigned* amax = reinterpret_cast<unsigned*>(scales);  // amax bits first, scales at the end
    if (cudaMemsetAsync(amax, 0, BH * d * sizeof(float), st) != cudaSuccess) return ATTN_ERR_CUDA;
    const dim3 grid((unsigned)((N + 127) / 128), (unsigned)BH);
    if (d == 128) {
      ta::channel_amax_kernel<128><<<grid, 256, 0, st>>>(x, amax, N);
      ta::channel_codes_kernel<128><<<grid, 256, 0, st>>>(x, amax, codes, N);
    } else {
      ta::channel_amax_kernel<64><<<grid, 256, 0, st>>>(x, amax, N);
      ta::channel_codes_kernel<64><<<grid, 256, 0, st>>>(x, amax, codes, N);
    }
    ta::channel_scale_kernel<<<(unsigned)((BH * d + 255) / 256), 256, 0, st>>>(amax, (int)(BH * d));
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_fwd_fp8(const uint8_t* q, const float* q_scale, const uint8_t* k, const float* k_scale, const uint8_t* v,
                 const float* v_scale, float* o, float* lse, int B, int H, int Nq, int Nkv, int d, int causal,
                 float scale, int rotated, void* stream) {
  if (B < 0 || H < 0 || Nq < 0 || Nkv < 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * H > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || Nq == 0) return ATTN_OK;
  if (Nkv == 0) return ATTN_ERR_UNSUPPORTED;
  if (!q || !q_scale || !k || !k_scale || !v || !v_scale || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(v_scale) ||
      !aligned4(q_scale) || !aligned4(k_scale) || !aligned4(lse))
    return ATTN_ERR_MISALIGNED;
  using C = ta::FwdF8Cfg;
  const int BH = B * H;
  CUtensorMap tq, tk, tv;
  int rc;
  if ((rc = make_tmap_i8(&tq, q, Nq, BH)) != ATTN_OK) return rc;
  if ((rc = make_tmap_i8(&tk, k, Nkv, BH)) != ATTN_OK) return rc;
  if ((rc = make_tmap_i8(&tv, v, Nkv, BH)) != ATTN_OK) return rc;
  if ((rc = set_smem_attr(ta::fwd_fp8_kernel, C::SMEM)) != ATTN_OK) return rc;
  ta::FwdF8Params p;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.o = o;
  p.lse = lse;
  p.Nq = Nq;
  p.Nkv = Nkv;
  p.n_qp = (Nq + 255) / 256;
  p.Tc = (Nkv + 127) / 128;
  p.causal = causal ? 1 : 0;
  p.ks_vec = (Nkv % 4 == 0) && aligned16(k_scale);
  p.sl2 = scale * 1.4426950408889634f / (rotated ? 128.f : 1.f);
  p.timeout_ns = g_wait_ns;
  const long long grid = (long long)BH * p.n_qp;
  if (grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  ta::fwd_fp8_kernel<<<(unsigned)grid, C::THREADS, C::SMEM, reinterpret_cast<cudaStream_t>(stream)>>>(tq, tk, tv,
                                                                                                     p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

size_t attn_nvfp4_codes_bytes(int B, int H, int N, int d, int mode) {
  if (B <= 0 || H <= 0 || N <= 0 || d != 128) return 0;
  const size_t BH = (size_t)B * H;
  return mode ? BH * 128 * (size_t)((N + 127) / 128) * 64 : BH * (size_t)N * 64;
}

size_t attn_nvfp4_sf_bytes(int B, int H, int N, int d, int mode) {
  if (B <= 0 || H <= 0 || N <= 0 || d != 128) return 0;
  (void)mode;  // both modes: one 1 KB block per 128-row (or 128-token) tile
  return (size_t)B * H * (size_t)((N + 127) / 128) * 1024;
}

int attn_quantize_nvfp4(const attn_bf16_t* x, uint8_t* codes, uint8_t* sf, int B, int H, int N, int d, int mode,
                        void* stream) {
  if (B < 0 || H < 0 || N < 0 || (mode != 0 && mode != 1)) return ATTN_ERR_INVALID_ARG;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || N == 0) return ATTN_OK;
  if (!x || !codes || !sf) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(sf)) return ATTN_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const long long BH = (long long)B * H;
  const int T = (N + 127) / 128;
  if (mode == 0) {
    const long long total = BH * T * 128 * 8;
    ta::quant_nvfp4_rows_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(x, codes, sf, N, T, total);
  } else {
    const long long total = BH * T * 8 * 128;
    ta::quant_nvfp4_cols_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(x, codes, sf, N, T, total);
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_fwd_fp4(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k, const uint8_t* k_sf, const uint8_t* vt,
                 const uint8_t* vt_sf, float* o, float* lse, int B, int H, int Nq, int Nkv, int d, int causal,
                 float scale, int p_mode, void* stream) {
  if (B < 0 || H < 0 || Nq < 0 || Nkv < 0 || (p_mode != 0 && p_mode != 1)) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * H > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || Nq == 0) return ATTN_OK;
  if (Nkv == 0) return ATTN_ERR_UNSUPPORTED;
  if (!q || !q_sf || !k || !k_sf || !vt || !vt_sf || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(vt) || !aligned16(q_sf) || !aligned16(k_sf) ||
      !aligned16(vt_sf) || !aligned16(o) || !aligned4(lse))
    return ATTN_ERR_MISALIGNED;
  return launch_fp4<false>(q, q_sf, k, k_sf, vt, vt_sf, o, lse, nullptr, B, H, Nq, Nkv, causal, scale, p_mode,
                           reinterpret_cast<cudaStream_t>(stream));
}

int attn_fp4_scores(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k, const uint8_t* k_sf, float* s, int B,
                    int H, int Nq, int Nkv, int d, void* stream) {
  if (B < 0 || H < 0 || Nq < 0 || Nkv < 0) return ATTN_ERR_INVALID_ARG;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || Nq == 0 || Nkv == 0) return ATTN_OK;
  if (!q || !q_sf || !k || !k_sf || !s) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_sf) || !aligned16(k_sf) || !aligned4(s))
    return ATTN_ERR_MISALIGNED;
  return launch_fp4<true>(q, q_sf, k, k_sf, nullptr, k_sf, nullptr, nullptr, s, B, H, Nq, Nkv, 0, 1.f, 0,
                          reinterpret_cast<cudaStream_t>(stream));
}

int attn_check_status(void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return ATTN_ERR_CUDA;
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, ta::g_attn_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  const int zero = 0;
  if (h != 0 && cudaMemcpyToSymbol(ta::g_attn_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  return h;
}

int attn_watchdog_selftest(unsigned long long limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return ATTN_ERR_INVALID_ARG;
  watchdog_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // extern "C"

int attn_debug_counters(unsigned long long* out, int reset) {
  if (!out) return ATTN_ERR_INVALID_ARG;
  if (!TA_DEBUG) return ATTN_ERR_UNSUPPORTED;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemcpyFromSymbol(out, ta::g_attn_counters, sizeof(unsigned long long) * ta::TA_NCOUNTERS) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (reset) {
    const unsigned long long zero[ta::TA_NCOUNTERS] = {};
    if (cudaMemcpyToSymbol(ta::g_attn_counters, zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}
