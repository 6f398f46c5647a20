/*
 * dmel_debug.h — diagnostics of the dMel library. Not part of the front end's data path: no
 * entry point of dmel.h calls these.
 */
#ifndef DMEL_DEBUG_H
#define DMEL_DEBUG_H

#include <stdint.h>

#include "dmel.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Runs, on the host, the same per-frame step functions the codes kernel runs on the device
 * (25 x 32 split of the 800-point complex DFT, real-signal split, sparse mel sums, log10,
 * clamp, quantise), lane after lane, for one already-framed block of 1600 samples
 * (frame1600 = x[800 (t-1) .. 800 (t+1))). Writes 80 codes and, when lhat80 != NULL, the 80
 * clamped log10 mel energies. Lets the kernel's arithmetic be checked without a GPU. */
void dmel_debug_codes_frame_host(const float *frame1600, uint8_t *codes80, double *lhat80);

/* The same with the level mapping q of dmel_codes_q (NULL: the default). Returns
 * DMEL_ERR_INVALID_ARG for a quantiser dmel_codes_q would reject. */
dmel_status dmel_debug_codes_frame_host_q(const float *frame1600, const dmel_quantizer *q, uint8_t *codes80,
                                          double *lhat80);

/* Failure-detection self test: launches one thread that waits, with a limit of `polls`
 * mbarrier polls, on a barrier phase that can never complete (two arrivals expected, one
 * made). The wait must give up and the kernel return; the call synchronises, then reads and
 * clears the device error word into *h_bits (DMEL_DEVERR_WAIT_TIMEOUT expected). Nothing
 * faults or hangs: the context stays usable. */
dmel_status dmel_debug_wait_timeout(uint32_t polls, uint32_t *h_bits);

/* y[i] = GELU(x[i]) for i < n with the formula the hMLP kernels use (u Phi(u), erfc from
 * Abramowitz & Stegun 7.1.26, absolute error at most 1.5e-7 in erfc), so it can be checked
 * against the exact function. x, y: device fp32 [n], 16-byte aligned. Asynchronous on stream. */
dmel_status dmel_debug_gelu(const float *x, float *y, int64_t n, dmel_stream_t stream);

/* The chunk plan dmel_forward_host follows for these host sample offsets (host only, pure).
 * Writes, chunk after chunk, into h_plan (at most cap int64 values):
 *   f0, f1          the chunk's frames [f0, f1) of the batch
 *   s_lo, s_hi      the host samples [s_lo, s_hi) it copies to the device
 *   tail            1 when its first piece starts inside its clip (the first 800 copied samples
 *                   are then that piece's tail, the rest its samples), else 0
 *   n               its number of pieces (one per clip with frames in the chunk)
 *   so[n + 1]       the pieces' sample offsets within the copied samples (after the tail)
 *   fo[n + 1]       the pieces' frame offsets within the chunk
 * *h_len receives the number of int64 values the whole plan needs (so a call with cap 0 sizes
 * it). Returns DMEL_ERR_INVALID_ARG for bad offsets or chunk_frames <= 0. */
dmel_status dmel_debug_forward_host_plan(const int64_t *h_sample_offsets, int n_clips, int64_t chunk_frames,
                                         int64_t *h_plan, int64_t cap, int64_t *h_len);

/* RMSNorm from the Gram matrix: the embedding's RMSNorm scales come from G = T T^T (the table's
 * 1280 x 1280 Gram matrix, fp32), because a frame's sum of squares is
 * sum_j x_j^2 = sum_b sum_b' G[16 b + c_b, 16 b' + c_b'].
 * dmel_debug_gram writes G for a bf16 table [1280 x embed_dim] (embed_dim a multiple of 128) into
 * the first half of the device array gram [2 x 1280 x 1280] (row-major; the 55 blocks of 128 x 128
 * entries whose row block is at most their column block are written, the others left as they
 * are; the second half is scratch), asynchronously on stream. dmel_debug_norm_sumsq_host evaluates, on the host, the sum of squares of one frame
 * with codes codes80 from a host copy of such a G, in the order the device sums it (blocks of
 * 8 x 8 bins in order, diagonal terms once, other pairs twice), into *h_sumsq. */
dmel_status dmel_debug_gram(const void *table, int embed_dim, float *gram, dmel_stream_t stream);
dmel_status dmel_debug_norm_sumsq_host(const uint8_t *codes80, const float *h_gram, double *h_sumsq);

/* The hMLP stage GEMM alone ("Inside Inkling: Audio Design", Part 1 · Modeling: each hMLP stage
 * is a linear map of the merged features): c [m x n] fp32 = a [m x k] bf16 (row stride lda
 * elements) times b [k x n] bf16, all row-major device arrays, fp32 sums, on the tcgen05 CTA-pair
 * kernel dmel_hmlp uses for stages 2-4. m >= 0; n, k and lda positive multiples of 8 with
 * lda >= k; a, b and c 16-byte aligned; m at most 2^31 - 1. Asynchronous on stream. */
dmel_status dmel_debug_gemm(const void *a, int64_t m, int k, int lda, const void *b, int n, float *c,
                            dmel_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DMEL_DEBUG_H */
