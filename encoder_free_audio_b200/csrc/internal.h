// Host-side interface between the library's translation units (not part of the C ABI).
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "dmel.h"

namespace dmel {

// The level mapping of the codes (dmel_quantizer, checked): clamp range, mode, mu, and the
// derived constants the kernel uses. Quant() is the default reading: [-7, 2], uniform floor.
struct Quant {
  float lmin = -7.0f, lmax = 2.0f, range = 9.0f;
  int mode = 0;  // 0 uniform floor, 1 nearest of 16 reconstruction points, 2 mu-law
  float mu = 0.0f, inv_log1p_mu = 0.0f;
};

// Codes of n_frames frames (and the carried tails when tails_out != nullptr) on `stream`.
// Adds the number of kernels launched to *launches.
cudaError_t launch_codes(const float *wav, const int64_t *soff, const int64_t *foff, int n_clips, int64_t n_frames,
                         const float *tails, float *tails_out, uint8_t *codes, uint32_t *err, int num_sms,
                         cudaStream_t stream, int *launches, Quant q = Quant());

// Whether the tensor-core embedding path takes this request.
bool embed_uses_tensor_cores(dmel_dtype table_dtype, int embed_dim);

// Scratch bytes the embedding needs (RMSNorm partial sums of the tensor-core path).
size_t embed_workspace_bytes(int64_t n_frames, int embed_dim, dmel_dtype table_dtype, int with_rmsnorm);

// Scratch the embedding needs when its RMSNorm scales come from an exchange of row sums between
// the CTAs of a row (no G): what dmel_embed_noalloc's fixed scratch must hold.
size_t embed_exchange_workspace_bytes(int64_t n_frames, int embed_dim, dmel_dtype table_dtype, int with_rmsnorm);

// Embedding of n_frames codes; workspace holds embed_workspace_bytes(...) bytes (with allow_gram
// false, embed_exchange_workspace_bytes(...)).
// out_rows: NULL (frame f -> row f of out) or device int64 [n_frames], frame f -> row out_rows[f]
// of an out with out_n_rows rows. gram: a table's G prepared beforehand (launch_gram), or NULL; with
// RMSNorm on a bf16 table it is used at every call size instead of computing G.
cudaError_t launch_embed(const uint8_t *codes, int64_t n_frames, const void *table, dmel_dtype table_dtype,
                         int embed_dim, const void *rms_weight, float eps, void *out, dmel_dtype out_dtype,
                         void *workspace, uint32_t *err, int num_sms, cudaStream_t stream, int *launches,
                         const int64_t *out_rows = nullptr, int64_t out_n_rows = 0, bool allow_gram = true,
                         const float *gram = nullptr);

// G = T T^T (fp32 [1280 x 1280], the 55 blocks of 128 x 128 rows with row block <= column block
// written; gram_bytes() holds it and a second partial product after it) of a bf16 table
// T [1280 x D], D a multiple of 128; and the RMSNorm scale of each frame,
// 1 / sqrt(sum_b sum_b' G[r_b, r_b'] / D + eps), from its codes (scratch: norm_scale_bytes(F)
// minus the F scales at its end); the scale kernels also set *zero_counter (when given) to 0.
size_t gram_bytes();
size_t norm_scale_bytes(int64_t n_frames);
cudaError_t launch_gram(const void *table, int D, float *G, uint32_t *err, cudaStream_t stream, int *launches);
cudaError_t launch_norm_scale(const uint8_t *codes, int64_t n_frames, int D, const float *G, float eps, void *scratch,
                              float *scale, int *zero_counter, int num_sms, cudaStream_t stream, int *launches);
double norm_sumsq_host(const uint8_t *codes80, const float *G);

// dmel_forward_host: workspace bytes for this batch (0 when it has no frame) and the pipelined
// run (host samples in, host vectors and codes out; streams and events of the library's own).
// *too_small is set (and nothing queued) when the workspace is smaller than the first reports.
size_t forward_host_workspace_bytes(const int64_t *h_sample_offsets, int n_clips, int embed_dim,
                                    dmel_dtype table_dtype, dmel_dtype out_dtype, int with_rmsnorm,
                                    int64_t chunk_frames);
cudaError_t run_forward_host(const float *h_wav, const int64_t *h_sample_offsets, int n_clips, const void *table,
                             dmel_dtype table_dtype, int embed_dim, const void *rms_weight, float eps, void *h_out,
                             dmel_dtype out_dtype, uint8_t *h_codes, int64_t chunk_frames, void *workspace,
                             size_t workspace_bytes, uint32_t *err, int num_sms, cudaStream_t stream, int *launches,
                             bool *too_small);
// The plan of run_forward_host flattened for dmel_debug_forward_host_plan; returns its length.
int64_t debug_forward_host_plan(const int64_t *h_sample_offsets, int n_clips, int64_t chunk_frames, int64_t *h_plan,
                                int64_t cap);

// Size of the fixed device scratch used by dmel_embed_noalloc.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;

// Device address of that scratch on the current device (looked up once per device).
cudaError_t noalloc_scratch(void **ptr);

// ShortConv of n_tokens tokens (sequences by device seq_offsets [n_seq + 1]) on `stream`: y, and
// the carried state out when state_out != nullptr (may be the state in). Adds the kernels
// launched to *launches.
cudaError_t launch_shortconv(const void *x, const int64_t *seq_offsets, int n_seq, int64_t n_tokens, int channels,
                             const float *weights, const void *state, void *state_out, void *y, dmel_dtype dtype,
                             uint32_t *err, int num_sms, cudaStream_t stream, int *launches);

// hMLP patchifier: workspace bytes for n_patches, and the launch on `stream` (stage 1 fused in
// one tcgen05 kernel when d1 is a multiple of 256, else gather + GEMM + row kernel; stages 2-4
// as cuBLASLt GEMMs + row kernels).
size_t hmlp_workspace_bytes(int64_t n_patches, const dmel_hmlp_weights &w);
cudaError_t launch_hmlp(const void *images, int n, int H, int W, const dmel_hmlp_weights &w, void *out,
                        void *workspace, uint32_t *err, int num_sms, cudaStream_t stream, int *launches);

// Raises a kernel's dynamic shared-memory limit to `bytes` once per device. `done` is that
// kernel's own flag array [256] (by device ordinal); concurrent first calls from several host
// threads may both set the attribute, which is harmless.
template <typename K>
cudaError_t set_smem_attr_once(K kernel, int bytes, std::atomic<bool> *done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (done[dev & 255].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[dev & 255].store(true, std::memory_order_release);
  return e;
}

// cuTensorMapEncodeTiled, looked up once from the driver (nullptr when unavailable).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

// GELU of n values with the hMLP kernels' formula (diagnostic).
cudaError_t launch_gelu_debug(const float *x, float *y, int64_t n, int num_sms, cudaStream_t stream);
cudaError_t launch_gemm_debug(const void *a, int64_t m, int k, int lda, const void *b, int n, float *c, uint32_t *err,
                              int num_sms, cudaStream_t stream);

// Launches a kernel whose bounded wait cannot be satisfied; *h_returned = 1 once it returned.
cudaError_t run_wait_timeout_selftest(uint32_t polls, uint32_t *err, int *h_returned);

void emulate_codes_frame_host(const float *frame1600, uint8_t *codes80, double *lhat80, Quant q = Quant());

}  // namespace dmel
