/*
 * tiledattn_probe -- throughput microbenchmarks that supply the roofline
 * denominators of the attention library on sm_100a.  Not part of the
 * attention path and with no counterpart on the pages: they measure the
 * hardware the kernels of libtiledattn run on.
 *
 *   tap_mma_rate   back-to-back tcgen05.mma from shared-memory operands into
 *                  tensor memory, one kind per call: the tensor-core ceiling
 *                  of that operand type (bf16, int8, e4m3, block-scaled e2m1).
 *   tap_ex2_rate   independent MUFU ex2.approx chains: exponentials per clock.
 *   tap_softmax_rate  the per-score work of the bf16 softmax (f32x2 FMA, two
 *                  ex2, f32x2 add, bf16x2 convert) per pair of scores.
 *
 * Conventions (as libtiledattn): device pointers owned by the caller, `stream`
 * is a cudaStream_t passed as void*, launches are asynchronous, the return
 * value is 0 or a negative status (-1 invalid argument, -4 CUDA launch error).
 * Every wait inside the MMA kernel is bounded (1 s); a wait that gives up
 * writes -5 into cycles[block] instead of a count (read it after a sync).
 *
 * Each call launches `grid` CTAs; CTA b writes the SM clock cycles its timed
 * loop took into cycles[b] (unsigned long long, `grid` entries).  With a grid
 * of one CTA per SM the rate per SM is (work per CTA) / cycles; the host
 * also times the launch with CUDA events to convert to per-second rates.
 */
#ifndef TILEDATTN_PROBE_H
#define TILEDATTN_PROBE_H

#ifdef __cplusplus
extern "C" {
#endif

/* MMA kinds */
#define TAP_KIND_BF16 0 /* kind::f16, bf16 x bf16 -> f32, K = 16 per instruction */
#define TAP_KIND_I8 1   /* kind::i8, s8 x s8 -> s32, K = 32 */
#define TAP_KIND_F8 2   /* kind::f8f6f4, e4m3 x e4m3 -> f32, K = 32 */
#define TAP_KIND_F4 3   /* kind::mxf4nvf4 block_scale scale_vec::4X, e2m1 x e2m1 with ue4m3
                           scales per 16 elements -> f32, K = 64 (N = 128 only) */

/* Variants (flags, OR-ed):
 *   TAP_A_TMEM       the A operand is read from tensor memory (the form the
 *                    attention kernels use for P V); not for TAP_KIND_F4
 *   TAP_TWO_ACC      one issuing thread alternates two independent
 *                    accumulators (n = 128)
 *   TAP_TWO_ISSUERS  two warps issue, each into its own accumulator, the
 *                    same `iters` x 4 MMAs each (n = 128; MACs per CTA double) */
#define TAP_A_TMEM 1
#define TAP_TWO_ACC 2
#define TAP_TWO_ISSUERS 4

/* Each CTA (128 threads, one per SM: 512 TMEM columns) issues `iters` x 4
 * MMAs of shape M = 128, N = `n` (128 or 256), K as above, accumulating in
 * tensor memory, B (and A unless TAP_A_TMEM) from 128-byte-swizzled shared
 * memory (e2m1: 64-byte), values drawn once and finite.  MACs per issuing
 * thread = iters * 4 * 128 * n * K; cycles[b] is the first issuer's.
 * Returns -1 for an unknown kind or flag, n not in {128, 256} (128 for
 * TAP_KIND_F4 and for the two-accumulator variants), iters < 1, grid < 1 or
 * a null `cycles`. */
int tap_mma_rate(int kind, int n, int iters, int grid, int flags, unsigned long long* cycles, void* stream);

/* The same measurement with the issue loop fixed at compile time: kind
 * (bf16, int8, e4m3; block-scaled e2m1 with n = 128 and no flag but
 * TAP_COMMIT, 64-byte swizzled tiles and unit scale factors as the FP4
 * attention kernel uses), N (128 or 256) and the A source as template
 * parameters, descriptors computed before the loop, `iters` groups of eight
 * MMAs (K = 256 bytes per row: the K sweep of a 128-deep tile pair) with
 * immediate offsets, all into one accumulator.  TAP_COMMIT adds a
 * tcgen05.commit to an mbarrier after every group, as the attention kernels
 * issue them.  MACs per CTA = iters * 8 * 128 * n * K. */
#define TAP_COMMIT 8
/* TAP_B_MN (n = 128): B stored MN-major (N contiguous), as the attention
 *   kernels read V for P V.  TAP_ATTN (n = 128): every group of eight
 *   K-major MMAs (S = Q K^T) is followed by eight with A from tensor memory
 *   and an MN-major B (O += P V) into a second accumulator, as one query
 *   tile's KV step; MACs per CTA double. */
#define TAP_B_MN 16
#define TAP_ATTN 32
/* With TAP_ATTN only: TAP_TESTWAIT tests a completed mbarrier
 *   (mbarrier.test_wait) before the last MMA of every group; TAP_WAITFENCE
 *   waits on it (the bounded try_wait loop) and issues
 *   tcgen05.fence::after_thread_sync before every pair of groups -- the
 *   barrier traffic of the attention kernels' issue thread. */
#define TAP_TESTWAIT 64
#define TAP_WAITFENCE 128
/* With TAP_ATTN only: warps 1-3 stream tcgen05.ld (128 columns) and
 *   tcgen05.st (64 columns) over tensor-memory columns [384, 512) of their
 *   lane quarters while the MMAs run, as the attention softmax does. */
#define TAP_TMEM_TRAFFIC 256
/* With TAP_ATTN only: TAP_FLAGPOLL loads a shared-memory word (already set)
 *   with ld.acquire before the last MMA of every S group; TAP_FLAGFENCE does
 *   that load and a tcgen05.fence::after_thread_sync before every pair of
 *   groups -- the same synchronisation points as TAP_TESTWAIT /
 *   TAP_WAITFENCE, through a plain flag instead of an mbarrier. */
#define TAP_FLAGPOLL 512
#define TAP_FLAGFENCE 1024
/* TAP_TWO_ISSUERS is accepted here together with TAP_ATTN (and optionally
 *   TAP_TESTWAIT | TAP_WAITFENCE): two warps each issue the attention pattern
 *   into their own accumulators (both groups with A from shared memory);
 *   MACs per CTA double again. */
int tap_mma_tight_rate(int kind, int n, int iters, int grid, int flags, unsigned long long* cycles,
                       void* stream);

/* `threads` per CTA (32..1024, a multiple of 32), each running `ilp` (1, 2,
 * 4 or 8) independent chains x <- ex2(-x) for `iters` steps: ex2 per CTA =
 * threads * ilp * iters.  `sink` (float, grid * threads) receives the chains'
 * sums so nothing is optimised away. */
int tap_ex2_rate(int threads, int ilp, int iters, int grid, unsigned long long* cycles, float* sink,
                 void* stream);

/* `threads` per CTA, each repeating for `iters` steps, on 8 pairs of scores:
 * (x0, x1) = fma.f32x2(s, scale, -m); p = ex2(x0), ex2(x1); l += (p0, p1)
 * (add.f32x2); w ^= cvt.rn.bf16x2(p0, p1).  Score pairs per CTA = threads * 8
 * * iters.  `sink` as above. */
int tap_softmax_rate(int threads, int iters, int grid, unsigned long long* cycles, float* sink, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* TILEDATTN_PROBE_H */
