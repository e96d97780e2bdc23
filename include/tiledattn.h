/*
 * tiledattn -- fused tiled scaled-dot-product attention forward for NVIDIA
 * B200 (sm_100a), C ABI.
 *
 * Sources, cited by page title and section:
 *   [FA-trading]   "Can a full-day context beat one minute? Flash attention and
 *                  the sequence-length question" (marketmaker.cc blog)
 *   [FA4-overview] "FlashAttention 4: fast, memory-saving attention for LLMs"
 *                  (linux-konsole)
 *   [FP4-FA4]      "Hardware-Aware FP4 FlashAttention-4" (gist.science summary)
 *   [INT-FA]       "INT-FlashAttention: an INT8 quantisation architecture
 *                  compatible with FlashAttention" (hoodcat.net)
 *
 * Conventions shared by every call
 *   - Tensor arguments are DEVICE pointers owned by the caller.  The library
 *     never allocates, frees or retains them.  Layout is contiguous row-major
 *     [B][H][N][d] (q, k, v shaped (batch, heads, seq, head_dim) as in
 *     [FA-trading] "Integration in eight lines"); LSE is [B][H][N_q].
 *   - bf16 tensors are passed as `attn_bf16_t` (the raw 16-bit pattern).
 *   - Tensor pointers must be 16-byte aligned (TMA and vector loads);
 *     float outputs 4-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous: the return value reports argument
 *     errors and launch errors only.  A device-side watchdog (every wait in a
 *     kernel has a time limit) reports ATTN_ERR_TIMEOUT through
 *     attn_check_status().
 *   - Causal semantics: key j is visible to query i iff j <= i + (N_kv - N_q)
 *     (the last query sees every key; for N_q == N_kv this is the usual
 *     lower-triangular mask, [FA-trading] "Causal masking").  A query row that
 *     sees no key gets O = 0 and LSE = -inf.
 *   - LSE is the natural-log log-sum-exp of the scaled scores of the row, the
 *     O(N) softmax statistic kept for the backward pass ([FA-trading]
 *     "Backward: recompute instead of store").
 *   - scale must be finite and > 0 (normally 1/sqrt(d)).
 *   - There is no fallback: an unsupported shape returns an error code.
 */
#ifndef TILEDATTN_H
#define TILEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

typedef uint16_t attn_bf16_t;

enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = -1, /* null pointer, negative size, bad scale      */
  ATTN_ERR_UNSUPPORTED = -2, /* head dim or shape outside what is built     */
  ATTN_ERR_MISALIGNED = -3,  /* pointer not 16-byte aligned                 */
  ATTN_ERR_CUDA = -4,        /* CUDA runtime/driver error at launch         */
  ATTN_ERR_TIMEOUT = -5,     /* a kernel wait ran past its time limit       */
  ATTN_ERR_TOO_LARGE = -6,   /* request needs more than the library's fixed
                                scratch (attn_decode_noalloc)               */
  ATTN_ERR_BOUNDS = -7       /* debug build only: a kernel's TMA coordinate
                                or tensor-memory address failed its check;
                                the access was skipped (attn_debug_counters) */
};

/* Human-readable name of a status code (static string). */
ATTN_API const char* attn_status_string(int status);

/* Library version, e.g. "tiledattn 0.1 sm_100a". */
ATTN_API const char* attn_version(void);

/*
 * attn_fwd -- bf16 attention forward, fp32 accumulation.
 *
 * [FA-trading] "The Flash Attention algorithm" (Q in B_r-row blocks, K/V in
 * B_c-column blocks, S_ij never leaves the chip), "Online softmax recurrence"
 * (running max m, running sum l, retroactive rescale of O), "FA2" (one
 * division by l after the inner loop; parallel over query blocks), "Causal
 * masking" (tiles entirely in the future are skipped); [FA4-overview]
 * "What is new in FlashAttention 4" (warp-specialised load / MMA / softmax /
 * correction / store roles) and "Smarter online softmax rescaling" (the
 * reference max only moves when it rises by more than 8 in log2 units).
 *
 *   q   [B][H][Nq][d]  bf16      k, v [B][H][Nkv][d] bf16
 *   o   [B][H][Nq][d]  bf16 out  lse  [B][H][Nq]     fp32 out (natural log)
 *   d in {64, 128}; Nq, Nkv >= 0 (Nq == 0 or B*H == 0: nothing to do;
 *   Nkv == 0: every row gets O = 0, LSE = -inf).
 */
ATTN_API int attn_fwd(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o,
             float* lse, int B, int H, int Nq, int Nkv, int d, int causal, float scale,
             void* stream);

/*
 * attn_fwd_gqa -- attn_fwd with grouped-query / multi-query attention:
 * Hq query heads share Hkv key/value heads, query head h reading key/value
 * head h / (Hq / Hkv) ([FA4-overview] "Compatibility and current status":
 * several attention heads use the same key/value projection, to save memory;
 * Hkv = 1 is multi-query attention, Hkv = Hq is attn_fwd).
 *
 *   q [B][Hq][Nq][d] bf16, k, v [B][Hkv][Nkv][d] bf16, o [B][Hq][Nq][d] bf16
 *   out, lse [B][Hq][Nq] fp32 out; Hkv >= 1 and Hq % Hkv == 0, else
 *   ATTN_ERR_INVALID_ARG.  Everything else as attn_fwd.
 */
ATTN_API int attn_fwd_gqa(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o,
                          float* lse, int B, int Hq, int Hkv, int Nq, int Nkv, int d, int causal, float scale,
                          void* stream);

/*
 * attn_bwd -- bf16 attention backward by recomputation ([FA-trading]
 * "Backward: recompute instead of store": P is never stored by the forward;
 * it is recomputed tile by tile from Q, K and the forward's softmax
 * statistics, here the LSE).  With S = scale Q K^T (masked as attn_fwd) and
 * P = exp(S - LSE):
 *   dV = P^T dO,  dP = dO V^T,  dS = P o (dP - rowsum(dO o O)),
 *   dQ = scale dS K,  dK = scale dS^T Q   (fp32 accumulation, bf16 out).
 *
 *   q, o, dout, dq [B][H][Nq][d] bf16; k, v, dk, dv [B][H][Nkv][d] bf16;
 *   lse [B][H][Nq] fp32 (attn_fwd's output for the same q, k, v, causal,
 *   scale); o = attn_fwd's O.  d in {64, 128}.  workspace: device scratch of
 *   at least attn_bwd_workspace_bytes(B, H, Nq) bytes, 16-byte aligned,
 *   owned by the caller (holds rowsum(dO o O)).  Nq == 0 or Nkv == 0: the
 *   gradients that exist are set to zero.
 */
ATTN_API size_t attn_bwd_workspace_bytes(int B, int H, int Nq);
ATTN_API int attn_bwd(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, const attn_bf16_t* o,
                      const attn_bf16_t* dout, const float* lse, attn_bf16_t* dq, attn_bf16_t* dk, attn_bf16_t* dv,
                      int B, int H, int Nq, int Nkv, int d, int causal, float scale, void* workspace,
                      size_t workspace_bytes, void* stream);

/*
 * attn_bwd_fp8p -- attn_bwd with the recomputed probabilities in 8-bit
 * floating point for the dV product ([FP4-FA4]: in training, 4-bit P made the
 * backward diverge, 8-bit P kept it stable): P = exp(S - LSE) is rounded to
 * e4m3 (round to nearest even, unit scale; P <= 1) before dV = P^T dO.
 * dS = P o (dP - Dr) uses P unrounded, so dQ and dK equal attn_bwd's.  Same
 * arguments, layouts and workspace as attn_bwd.
 */
ATTN_API int attn_bwd_fp8p(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, const attn_bf16_t* o,
                           const attn_bf16_t* dout, const float* lse, attn_bf16_t* dq, attn_bf16_t* dk,
                           attn_bf16_t* dv, int B, int H, int Nq, int Nkv, int d, int causal, float scale,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_decode -- split-KV decode: ONE query row per (batch, head) against a
 * KV cache of Nkv keys; the key range is cut into num_splits equal chunks of
 * ceil(Nkv / num_splits) keys, each chunk gives a partial (O_c, LSE_c) in the
 * workspace, and a combine kernel merges them:
 *   LSE = log sum_c exp(LSE_c),  O = sum_c exp(LSE_c - LSE) O_c.
 * The merge is the online-softmax identity ([FA-trading] "Online softmax
 * recurrence") applied to whole chunks.
 *
 *   q [B][H][1][d] bf16, k, v [B][H][Nkv][d] bf16, o [B][H][1][d] bf16 out,
 *   lse [B][H] fp32 out; d in {64, 128}; 1 <= num_splits <= 1024; Nkv >= 1.
 *   workspace: device scratch of at least attn_decode_workspace_bytes(...)
 *   bytes, 16-byte aligned, owned by the caller; its contents on entry do not
 *   matter and are overwritten.  Calls that share a workspace must not
 *   overlap in time.
 */
ATTN_API size_t attn_decode_workspace_bytes(int B, int H, int d, int num_splits);
ATTN_API int attn_decode(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o,
                float* lse, int B, int H, int Nkv, int d, float scale, int num_splits,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_decode_gqa -- attn_decode with Hq query heads sharing Hkv key/value
 * heads (query head h reads cache head h / (Hq / Hkv), as attn_fwd_gqa).
 * The query heads of a group are scheduled together, so the cache of a
 * key/value head crosses HBM once for the whole group.
 *
 *   q [B][Hq][1][d], k, v [B][Hkv][Nkv][d], o [B][Hq][1][d], lse [B][Hq];
 *   workspace: attn_decode_workspace_bytes(B, Hq, d, num_splits) bytes.
 *   Hkv >= 1 and Hq % Hkv == 0, else ATTN_ERR_INVALID_ARG; everything else as
 *   attn_decode.
 */
ATTN_API int attn_decode_gqa(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o,
                             float* lse, int B, int Hq, int Hkv, int Nkv, int d, float scale, int num_splits,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_fwd_varlen -- attn_fwd over a batch of sequences of different lengths
 * packed without padding ([FA4-overview] "Compatibility and current status":
 * variable-length batches).  Sequence b owns query rows
 * [cu_seqlens_q[b], cu_seqlens_q[b+1]) and keys [cu_seqlens_k[b],
 * cu_seqlens_k[b+1]); it attends only to its own keys, with the causal rule
 * of this header applied per sequence (N_q, N_kv = its own lengths).
 *   q, o  bf16 [total_q][H][d]   (token-major packing, 16-byte aligned)
 *   k, v  bf16 [total_k][Hkv][d] (grouped-query when Hkv < H; H % Hkv == 0)
 *   lse   fp32 [H][total_q]
 *   cu_seqlens_q, cu_seqlens_k  int32 [B + 1] DEVICE arrays, non-decreasing,
 *         starting at 0 (offsets are clamped to [0, total] on the device).
 *   max_seqlen_q  >= every sequence's query length (sets the grid; rows of a
 *         longer sequence past it are not written).
 *   Rows outside every sequence are not written.  A sequence with no keys
 *   gets O = 0, LSE = -inf.  d in {64, 128}.
 */
ATTN_API int attn_fwd_varlen(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o,
                             float* lse, const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H, int Hkv,
                             int total_q, int total_k, int max_seqlen_q, int d, int causal, float scale,
                             void* stream);

/*
 * attn_decode_varlen -- attn_decode_gqa with a cache length per batch entry
 * (variable-length batches, as attn_fwd_varlen): batch b attends to keys
 * [0, seqlens_k[b]) of its cache (clamped to [0, Nkv_max]); each entry's
 * keys are split into num_splits chunks of its own length.  An entry with no
 * keys gets O = 0, LSE = -inf.
 *   q [B][H][1][d], k/v [B][Hkv][Nkv_max][d] bf16, seqlens_k int32 [B] DEVICE
 *   array; o, lse, workspace as attn_decode.
 */
ATTN_API int attn_decode_varlen(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v, attn_bf16_t* o,
                                float* lse, const int* seqlens_k, int B, int H, int Hkv, int Nkv_max, int d,
                                float scale, int num_splits, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * attn_decode_noalloc -- the same split-KV decode as attn_decode, for callers
 * that cannot allocate device memory: code that runs where cudaMalloc is not
 * allowed or not wanted (inside a caller's own memory pool or allocator hook,
 * a plug-in with no allocator of its own, a latency-critical path that must
 * never enter the driver's allocator).  The pages have no counterpart: this
 * is a packaging variant, not part of the method.
 *
 * The per-split partial results live in one fixed device array inside the
 * library, ATTN_DECODE_NOALLOC_SCRATCH_BYTES (20 MiB) in size.  Every GPU that
 * loads the library holds that array until the process exits.  A request
 * whose partials need more than that -- B*H*num_splits*(d+1)*4 bytes plus
 * alignment, as attn_decode_workspace_bytes() reports -- is rejected with
 * ATTN_ERR_TOO_LARGE before anything is launched (the decode workload
 * B=64, H=32, d=128, 16 splits needs 16.1 MiB and fits).
 *
 * The function calls no allocator (no cudaMalloc/cudaFree, no library
 * routine that allocates).  The first call on a device looks up the device
 * address of the array with cudaGetSymbolAddress while that device is
 * current; make that first call before any stream capture.  All calls share
 * the array and it keeps the last call's contents; every partial is written
 * before it is read, so nothing needs clearing between calls.  Calls that
 * overlap on the GPU (different streams, or different host threads) race on
 * the array and must be serialised by the caller.
 *
 * Arguments, layouts and errors otherwise as attn_decode.
 */
#define ATTN_DECODE_NOALLOC_SCRATCH_BYTES (20u * 1024u * 1024u)
ATTN_API int attn_decode_noalloc(const attn_bf16_t* q, const attn_bf16_t* k, const attn_bf16_t* v,
                                 attn_bf16_t* o, float* lse, int B, int H, int Nkv, int d, float scale,
                                 int num_splits, void* stream);

/*
 * attn_quantize_int8 -- symmetric INT8 quantisation of a bf16 tensor
 * [B][H][N][d] ([INT-FA]: token-level post-training quantisation of Q, K, V).
 *   per_head == 0: one scale per token row, xs [B][H][N]   (Q and K);
 *   per_head != 0: one scale per (batch, head), xs [B][H] (V: P V contracts
 *                  over tokens, so V's scale must be shared by a head's tokens).
 * s = amax / 127 (IEEE fp32 divide; amax == 0 gives s = 1),
 * xq = clamp(rne(x / s), -127, 127) (IEEE divide, round to nearest even).
 *   x bf16 16-byte aligned, xq int8 [B][H][N][d] 16-byte aligned, xs fp32.
 *   d in {64, 128}.
 */
ATTN_API int attn_quantize_int8(const attn_bf16_t* x, int8_t* xq, float* xs, int B, int H, int N, int d,
                                int per_head, void* stream);

/*
 * attn_quantize_int4 -- token-level INT4 quantisation of Q or K ([INT-FA]:
 * the token-level scheme carries over to lower formats such as 4-bit
 * integers): one scale per token row, s = amax / 7 (IEEE fp32 divide;
 * amax == 0 gives s = 1), xq = clamp(rne(x / s), -7, 7), stored one code per
 * byte (int8 containers: attn_fwd_int8 consumes them unchanged, with V
 * quantised by attn_quantize_int8 per head).
 *   x bf16 [B][H][N][d] 16-byte aligned, xq int8 [B][H][N][d] 16-byte aligned,
 *   xs fp32 [B][H][N]; d in {64, 128}.
 */
ATTN_API int attn_quantize_int4(const attn_bf16_t* x, int8_t* xq, float* xs, int B, int H, int N, int d,
                                void* stream);

/*
 * attn_fwd_int8 -- INT8 attention forward ([INT-FA]: INT8 GEMMs for Q K^T and
 * P V inside the FlashAttention forward, int32 accumulation):
 *   S = q_i8 . k_i8 (int32, exact); x = S * q_scale[i] * k_scale[j] * scale;
 *   running row max moved on every increase; P8 = rne(127 * exp(x - m)) in
 *   [0, 127]; O accumulates P8 . v_i8 in int32 per block and in fp32 across
 *   max changes, times v_scale / 127; l sums P8 / 127; O = acc / l,
 *   LSE = m + ln l.
 *   q [B][H][Nq][128] int8 + q_scale [B][H][Nq]; k [B][H][Nkv][128] int8 +
 *   k_scale [B][H][Nkv]; v [B][H][Nkv][128] int8 + v_scale [B][H];
 *   o [B][H][Nq][128] fp32 out, lse [B][H][Nq] fp32 out.
 *   d must be 128; Nkv >= 1.
 */
ATTN_API int attn_fwd_int8(const int8_t* q, const float* q_scale, const int8_t* k, const float* k_scale,
                           const int8_t* v, const float* v_scale, float* o, float* lse, int B, int H, int Nq,
                           int Nkv, int d, int causal, float scale, void* stream);

/*
 * attn_int8_scores -- the int32 score tiles S = q_i8 k_i8^T of the INT8
 * forward, computed by the same tensor-core MMA path and written to
 * s [B][H][Nq][Nkv] int32 (a check of the integer GEMM; small sizes).
 */
ATTN_API int attn_int8_scores(const int8_t* q, const int8_t* k, int32_t* s, int B, int H, int Nq, int Nkv, int d,
                              void* stream);

/*
 * NVFP4 operands ([FP4-FA4]: FP4 Q, K, V on the FP4 tensor cores).
 * Blocks of 16 elements, e2m1 codes (RNE, saturating at +-6) with one unsigned
 * e4m3 scale per block: sf = e4m3_rne(amax / 6), code = e2m1_rne(x / sf)
 * (IEEE fp32 divides; a zero block gets scale 0 and codes 0).  Two codes per
 * byte, the lower-index element in the low nibble.  d must be 128.
 *   mode 0 (Q, K): blocks run along d; codes [B][H][N][64 bytes];
 *   mode 1 (V):    blocks run along tokens (P V contracts over tokens) and the
 *                  codes are written transposed, [B][H][128][ceil(N/128)*64
 *                  bytes] (tokens padded to a multiple of 128 with zeros).
 * Scales: one 1 KB block per 128 rows (mode 0) or per 128 tokens (mode 1),
 * [B][H][ceil(N/128)][1024 bytes], byte (r % 32) * 16 + (r / 32) * 4 + (b % 4)
 * + (b / 4) * 512 for row (mode 1: channel) r of the tile and block b (0..7)
 * -- the order in which the tensor core reads block scales.
 * attn_nvfp4_codes_bytes / attn_nvfp4_sf_bytes give the buffer sizes (0 for
 * an unsupported shape).
 */
ATTN_API size_t attn_nvfp4_codes_bytes(int B, int H, int N, int d, int mode);
ATTN_API size_t attn_nvfp4_sf_bytes(int B, int H, int N, int d, int mode);
ATTN_API int attn_quantize_nvfp4(const attn_bf16_t* x, uint8_t* codes, uint8_t* sf, int B, int H, int N, int d,
                                 int mode, void* stream);

/*
 * attn_fwd_fp4 -- FP4 attention forward with block-scaled FP4 tensor-core
 * MMAs for Q K^T and P V ([FP4-FA4]).  P is encoded either with Direct-P
 * (p_mode 0: the score maps straight to the e2m1 code of 6 * exp(x - m),
 * every P block scale 1) or quantised after the exponential (p_mode 1: per
 * 16 keys, sf = e4m3_rne(amax(p) / 6), code = e2m1_rne(p / sf)).  The running
 * max moves on every increase; l sums the dequantised P (divided by 6 for
 * Direct-P); O = acc / l (fp32), LSE = m + ln l.
 *   q, k: mode-0 codes + scales of Q [B][H][Nq][128], K [B][H][Nkv][128];
 *   vt, vt_sf: mode-1 codes + scales of V; o [B][H][Nq][128] fp32 out,
 *   lse [B][H][Nq] fp32 out.  d must be 128; Nkv >= 1.
 */
ATTN_API int attn_fwd_fp4(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k, const uint8_t* k_sf,
                          const uint8_t* vt, const uint8_t* vt_sf, float* o, float* lse, int B, int H, int Nq,
                          int Nkv, int d, int causal, float scale, int p_mode, void* stream);

/*
 * attn_fp4_scores -- S = deq(q) deq(k)^T (fp32, [B][H][Nq][Nkv]) through the
 * same block-scaled tensor-core path as attn_fwd_fp4 (a check of the FP4
 * GEMM; small sizes).
 */
ATTN_API int attn_fp4_scores(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k, const uint8_t* k_sf, float* s,
                             int B, int H, int Nq, int Nkv, int d, void* stream);

/*
 * FP8 (e4m3) operands with incoherent processing ([FA-trading] "FA2"/"FA3"
 * list, item 3: FP8 doubles the matmul rate; Q and K are rotated by a random
 * Hadamard transform before quantisation so that outliers spread over the
 * coordinates).  e4m3: OCP E4M3 (bias 7, largest finite 448), round to
 * nearest even, saturating; codes stored one per byte.
 * attn_quantize_fp8
 *   mode 0 (Q, K): one fp32 scale per token row.  If `signs` (fp32 [d], each
 *     +1 or -1, device) is given, the row is first rotated, y = H_d (signs o x)
 *     with H_d the unnormalised Sylvester Hadamard matrix, evaluated as the
 *     fast Walsh-Hadamard transform in fp32 (stages h = 1, 2, ..., d/2, pair
 *     (a, b) -> (a + b, a - b)); signs = NULL quantises x unrotated.
 *     s = amax(|y|) / 448 (IEEE fp32 divide; amax == 0 gives s = 1), codes
 *     e4m3(y / s); scales [B][H][N].
 *   mode 1 (V): one scale per (batch, head, channel) over the N tokens, no
 *     rotation; scales [B][H][d].
 *   x bf16 [B][H][N][d], codes [B][H][N][d] bytes (both 16-byte aligned);
 *   d in {64, 128}.
 */
ATTN_API int attn_quantize_fp8(const attn_bf16_t* x, uint8_t* codes, float* scales, int B, int H, int N, int d,
                               int mode, const float* signs, void* stream);

/*
 * attn_fwd_fp8 -- FP8 attention forward on the FP8 tensor cores
 * ([FA-trading] FA3 list item 3; tiling and online softmax as attn_fwd):
 *   S = codes(q) codes(k)^T (fp32 accumulation of exact e4m3 products);
 *   x = S * q_scale[i] * k_scale[j] * scale * log2(e) / r, r = d when q and k
 *   were rotated (rotated != 0: the rotation multiplies q k^T by d), else 1;
 *   per block of 128 keys a reference row max m moves to the block max only
 *   when that exceeds it by more than 8 (lazy rescaling, [FA4-overview]
 *   "Smarter online softmax rescaling"), P~ = e4m3(2^(x - m)) (values in
 *   [0, 256], unit scale), l = l 2^(m_old - m) + sum P~,
 *   acc = acc 2^(m_old - m) + P~ codes(v);
 *   O[i][c] = acc[i][c] * v_scale[c] / l (fp32), LSE = ln 2 (m + log2 l).
 *   q [B][H][Nq][128] codes + q_scale [B][H][Nq]; k [B][H][Nkv][128] codes +
 *   k_scale [B][H][Nkv]; v [B][H][Nkv][128] codes + v_scale [B][H][128]
 *   (16-byte aligned); o [B][H][Nq][128] fp32 out, lse [B][H][Nq] fp32 out.
 *   d must be 128; Nkv >= 1.
 */
ATTN_API int attn_fwd_fp8(const uint8_t* q, const float* q_scale, const uint8_t* k, const float* k_scale,
                          const uint8_t* v, const float* v_scale, float* o, float* lse, int B, int H, int Nq,
                          int Nkv, int d, int causal, float scale, int rotated, void* stream);

/*
 * attn_check_status -- synchronise `stream`, read the device status word
 * written by the kernels' watchdog (ATTN_OK or ATTN_ERR_TIMEOUT; in the debug
 * build also ATTN_ERR_BOUNDS), clear it and return it; also returns
 * ATTN_ERR_CUDA if the synchronisation itself fails.
 */
ATTN_API int attn_check_status(void* stream);

/*
 * attn_set_wait_limit_ns -- time limit of every in-kernel wait (default
 * 1e9 ns).  Applies to launches made after the call.  0 restores the default.
 */
ATTN_API void attn_set_wait_limit_ns(unsigned long long ns);

/*
 * attn_watchdog_selftest -- launch one CTA that waits on a barrier nothing
 * ever arrives at, with a limit of `limit_ns`.  The wait gives up, the kernel
 * records ATTN_ERR_TIMEOUT and returns normally; attn_check_status() then
 * reports it.  Exercises the timeout path without a fault or a hang.
 */
ATTN_API int attn_watchdog_selftest(unsigned long long limit_ns, void* stream);

/*
 * attn_debug_counters -- counters of the debug build (libtiledattn_debug.so,
 * compiled with TA_DEBUG = 1): the product build returns
 * ATTN_ERR_UNSUPPORTED and writes nothing.  Synchronises the device, copies
 * four unsigned 64-bit counters to `out` (host memory, 4 entries) and, if
 * `reset` is non-zero, clears them:
 *   out[0]  lazy rescales of the bf16 forward: query rows whose reference max
 *           moved (block max above it by more than 8 in log2 units) after
 *           the row's first key block ("FlashAttention 4" page, smarter
 *           online softmax rescaling), summed over launches;
 *   out[1]  key tiles that causal bf16-forward CTAs skipped (tiles wholly in
 *           the future of a query tile; "Can a full-day context beat one
 *           minute?" page, causal masking);
 *   out[2]  bounds violations: TMA coordinates or tensor-memory addresses
 *           that failed the debug build's checks (each also records
 *           ATTN_ERR_BOUNDS for attn_check_status and skips the access);
 *   out[3]  reserved (0).
 * Returns ATTN_ERR_INVALID_ARG for a null `out`, ATTN_ERR_CUDA if the copy
 * fails.
 */
ATTN_API int attn_debug_counters(unsigned long long* out, int reset);

#ifdef __cplusplus
}
#endif
#endif /* TILEDATTN_H */
