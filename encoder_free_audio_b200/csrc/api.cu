// C ABI of the dMel front end: argument checks, workspace layout and dispatch to the kernels.
#include <cmath>
#include <cstring>
#include <mutex>

#include "dmel.h"
#include "common.cuh"
#include "dmel_debug.h"
#include "internal.h"

namespace dmel {
namespace {

__device__ uint32_t d_error_word;

thread_local int t_last_launches = 0;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int major = 0;
  uint32_t *err = nullptr;
};
std::mutex g_dev_mu;
DeviceInfo g_dev[256];

// Per-device facts, looked up once: SM count, compute capability, address of the error word.
cudaError_t device_info(DeviceInfo *out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.ready) {
    if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return e;
    void *p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, d_error_word)) != cudaSuccess) return e;
    d.err = static_cast<uint32_t *>(p);
    d.ready = true;
  }
  *out = d;
  return cudaSuccess;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool dtype_ok(dmel_dtype t) { return t == DMEL_F32 || t == DMEL_BF16; }

// Checks of the embedding arguments; check_codes = false when the codes buffer is the
// library's own (dmel_forward without codes_out).
dmel_status check_embed_args(const uint8_t *codes, bool check_codes, int64_t n_frames, const void *table,
                             dmel_dtype table_dtype, int D, const void *rms_weight, float eps, const void *out,
                             dmel_dtype out_dtype) {
  if (n_frames < 0 || D <= 0 || D % 8 != 0) return DMEL_ERR_INVALID_ARG;
  if (!dtype_ok(table_dtype) || !dtype_ok(out_dtype)) return DMEL_ERR_INVALID_ARG;
  if (n_frames == 0) return DMEL_OK;
  if (!table || !out) return DMEL_ERR_INVALID_ARG;
  if (check_codes && (codes == nullptr || !aligned(codes, 16))) return DMEL_ERR_INVALID_ARG;
  if (rms_weight && !(eps > 0.0f)) return DMEL_ERR_INVALID_ARG;
  // 16-byte vector access of rows: table, weight and output bases 16-byte aligned; codes rows
  // (80 bytes) read as 16-byte vectors by the tensor-core path.
  if (!aligned(table, 16) || !aligned(out, 16) || (rms_weight && !aligned(rms_weight, 16)))
    return DMEL_ERR_INVALID_ARG;
  if (!embed_uses_tensor_cores(table_dtype, D) && D > 16384) return DMEL_ERR_INVALID_ARG;
  return DMEL_OK;
}

dmel_status check_codes_args(const float *wav, const int64_t *sample_offsets, const int64_t *frame_offsets,
                             int n_clips, int64_t n_frames, const uint8_t *codes) {
  if (n_clips < 0 || n_frames < 0) return DMEL_ERR_INVALID_ARG;
  if (n_clips == 0 && n_frames > 0) return DMEL_ERR_INVALID_ARG;
  if (n_clips == 0) return DMEL_OK;
  if (!sample_offsets || !frame_offsets) return DMEL_ERR_INVALID_ARG;
  if (n_frames > 0 && (!wav || !codes)) return DMEL_ERR_INVALID_ARG;
  return DMEL_OK;
}

dmel_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DMEL_OK : DMEL_ERR_CUDA; }

// dmel_quantizer -> Quant (NULL: the default); false for a quantiser the ABI rejects.
bool to_quant(const dmel_quantizer *q, Quant *out) {
  Quant z;
  if (q) {
    if (!std::isfinite(q->min_value) || !std::isfinite(q->max_value) || !(q->max_value > q->min_value)) return false;
    if (q->mode != DMEL_QUANT_FLOOR && q->mode != DMEL_QUANT_ROUND && q->mode != DMEL_QUANT_MULAW) return false;
    if (q->mode == DMEL_QUANT_MULAW && !(std::isfinite(q->mu) && q->mu > 0.0f)) return false;
    z.lmin = q->min_value;
    z.lmax = q->max_value;
    z.range = q->max_value - q->min_value;
    z.mode = q->mode;
    z.mu = q->mode == DMEL_QUANT_MULAW ? q->mu : 0.0f;
    z.inv_log1p_mu = q->mode == DMEL_QUANT_MULAW ? (float)(1.0 / std::log1p((double)q->mu)) : 0.0f;
    if (!std::isfinite(z.range)) return false;
  }
  *out = z;
  return true;
}

}  // namespace
}  // namespace dmel

using namespace dmel;

extern "C" {

int64_t dmel_frames_for_length(int64_t n_samples) { return n_samples < 0 ? -1 : n_samples / kHop; }

dmel_status dmel_frame_offsets(const int64_t *h_sample_offsets, int n_clips, int64_t *h_frame_offsets) {
  if (!h_sample_offsets || !h_frame_offsets || n_clips < 0) return DMEL_ERR_INVALID_ARG;
  if (h_sample_offsets[0] != 0) return DMEL_ERR_INVALID_ARG;
  int64_t acc = 0;
  for (int c = 0; c < n_clips; ++c)
    if (h_sample_offsets[c + 1] < h_sample_offsets[c]) return DMEL_ERR_INVALID_ARG;
  h_frame_offsets[0] = 0;
  for (int c = 0; c < n_clips; ++c) {
    acc += dmel_frames_for_length(h_sample_offsets[c + 1] - h_sample_offsets[c]);
    h_frame_offsets[c + 1] = acc;
  }
  return DMEL_OK;
}

size_t dmel_workspace_size(int64_t n_frames, int embed_dim, dmel_dtype table_dtype, int with_rmsnorm,
                           int with_codes_out) {
  if (n_frames <= 0 || embed_dim <= 0) return 0;
  size_t bytes = 0;
  if (!with_codes_out) bytes += round_up((size_t)n_frames * kMel, 256);
  bytes += round_up(embed_workspace_bytes(n_frames, embed_dim, table_dtype, with_rmsnorm), 256);
  return bytes;
}

dmel_status dmel_codes_q(const float *wav, const int64_t *sample_offsets, const int64_t *frame_offsets, int n_clips,
                         int64_t n_frames, const float *tails, float *tails_out, uint8_t *codes,
                         const dmel_quantizer *q, dmel_stream_t stream) {
  t_last_launches = 0;
  Quant qz;
  if (!to_quant(q, &qz)) return DMEL_ERR_INVALID_ARG;
  dmel_status st = check_codes_args(wav, sample_offsets, frame_offsets, n_clips, n_frames, codes);
  if (st != DMEL_OK || n_clips == 0) return st;
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) return DMEL_ERR_CUDA;
  if (d.major != 10) return DMEL_ERR_UNSUPPORTED;
  int launches = 0;
  cudaError_t e = launch_codes(wav, sample_offsets, frame_offsets, n_clips, n_frames, tails, tails_out, codes, d.err,
                               d.sms, reinterpret_cast<cudaStream_t>(stream), &launches, qz);
  t_last_launches = launches;
  return from_cuda(e);
}

dmel_status dmel_codes(const float *wav, const int64_t *sample_offsets, const int64_t *frame_offsets, int n_clips,
                       int64_t n_frames, const float *tails, float *tails_out, uint8_t *codes, dmel_stream_t stream) {
  return dmel_codes_q(wav, sample_offsets, frame_offsets, n_clips, n_frames, tails, tails_out, codes, nullptr, stream);
}

namespace {
// The table's G from dmel_table_prepare, when it applies to this call (RMSNorm on a bf16 table the
// tensor-core path takes); NULL otherwise. A misaligned pointer is an argument error (*bad).
const float *prepared_gram(const void *prepared, dmel_dtype table_dtype, int embed_dim, const void *rms_weight,
                           bool *bad) {
  *bad = prepared && !aligned(prepared, 256);
  if (!prepared || *bad || !rms_weight || dmel_table_prepare_size(embed_dim, table_dtype) == 0) return nullptr;
  return static_cast<const float *>(prepared);
}

dmel_status embed_rows_impl(const uint8_t *codes, int64_t n_frames, const void *table, dmel_dtype table_dtype,
                            int embed_dim, const void *rms_weight, float eps, const void *prepared, void *out,
                            const int64_t *out_rows, int64_t out_n_rows, dmel_dtype out_dtype, void *workspace,
                            size_t workspace_bytes, dmel_stream_t stream) {
  t_last_launches = 0;
  dmel_status st =
      check_embed_args(codes, true, n_frames, table, table_dtype, embed_dim, rms_weight, eps, out, out_dtype);
  if (st != DMEL_OK) return st;
  if (out_rows && (out_n_rows <= 0 || !aligned(out_rows, 8))) return DMEL_ERR_INVALID_ARG;
  if (n_frames == 0) return DMEL_OK;
  const size_t need = embed_workspace_bytes(n_frames, embed_dim, table_dtype, rms_weight != nullptr);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256))) return DMEL_ERR_INVALID_ARG;
  bool bad = false;
  const float *G = prepared_gram(prepared, table_dtype, embed_dim, rms_weight, &bad);
  if (bad) return DMEL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) return DMEL_ERR_CUDA;
  if (d.major != 10) return DMEL_ERR_UNSUPPORTED;
  int launches = 0;
  cudaError_t e = launch_embed(codes, n_frames, table, table_dtype, embed_dim, rms_weight, eps, out, out_dtype,
                               workspace, d.err, d.sms, reinterpret_cast<cudaStream_t>(stream), &launches, out_rows,
                               out_n_rows, true, G);
  t_last_launches = launches;
  return from_cuda(e);
}
}  // namespace

dmel_status dmel_embed_rows(const uint8_t *codes, int64_t n_frames, const void *table, dmel_dtype table_dtype,
                            int embed_dim, const void *rms_weight, float eps, void *out, const int64_t *out_rows,
                            int64_t out_n_rows, dmel_dtype out_dtype, void *workspace, size_t workspace_bytes,
                            dmel_stream_t stream) {
  return embed_rows_impl(codes, n_frames, table, table_dtype, embed_dim, rms_weight, eps, nullptr, out, out_rows,
                         out_n_rows, out_dtype, workspace, workspace_bytes, stream);
}

dmel_status dmel_embed_prepared(const uint8_t *codes, int64_t n_frames, const void *table, dmel_dtype table_dtype,
                                int embed_dim, const void *rms_weight, float eps, const void *prepared, void *out,
                                dmel_dtype out_dtype, void *workspace, size_t workspace_bytes, dmel_stream_t stream) {
  return embed_rows_impl(codes, n_frames, table, table_dtype, embed_dim, rms_weight, eps, prepared, out, nullptr, 0,
                         out_dtype, workspace, workspace_bytes, stream);
}

dmel_status dmel_embed(const uint8_t *codes, int64_t n_frames, const void *table, dmel_dtype table_dtype, int embed_dim,
                       const void *rms_weight, float eps, void *out, dmel_dtype out_dtype, void *workspace,
                       size_t workspace_bytes, dmel_stream_t stream) {
  return dmel_embed_rows(codes, n_frames, table, table_dtype, embed_dim, rms_weight, eps, out, nullptr, 0, out_dtype,
                         workspace, workspace_bytes, stream);
}

namespace {
dmel_status forward_rows_impl(const float *wav, const int64_t *sample_offsets, const int64_t *frame_offsets,
                              int n_clips, int64_t n_frames, const float *tails, float *tails_out, const void *table,
                              dmel_dtype table_dtype, int embed_dim, const void *rms_weight, float eps,
                              const void *prepared, void *out, const int64_t *out_rows, int64_t out_n_rows,
                              dmel_dtype out_dtype, uint8_t *codes_out, void *workspace, size_t workspace_bytes,
                              dmel_stream_t stream) {
  t_last_launches = 0;
  if (n_clips < 0 || n_frames < 0 || (n_clips == 0 && n_frames > 0)) return DMEL_ERR_INVALID_ARG;
  if (out_rows && (out_n_rows <= 0 || !aligned(out_rows, 8))) return DMEL_ERR_INVALID_ARG;
  if (!sample_offsets && n_clips > 0) return DMEL_ERR_INVALID_ARG;
  if (!frame_offsets && n_clips > 0) return DMEL_ERR_INVALID_ARG;
  if (n_frames > 0 && !wav) return DMEL_ERR_INVALID_ARG;
  dmel_status st = check_embed_args(codes_out, codes_out != nullptr, n_frames, table, table_dtype, embed_dim,
                                    rms_weight, eps, out, out_dtype);
  if (st != DMEL_OK) return st;
  if (n_clips == 0) return DMEL_OK;
  const size_t need = dmel_workspace_size(n_frames, embed_dim, table_dtype, rms_weight != nullptr, codes_out != nullptr);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256))) return DMEL_ERR_INVALID_ARG;
  bool bad = false;
  const float *G = prepared_gram(prepared, table_dtype, embed_dim, rms_weight, &bad);
  if (bad) return DMEL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) return DMEL_ERR_CUDA;
  if (d.major != 10) return DMEL_ERR_UNSUPPORTED;
  uint8_t *codes = codes_out;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  if (!codes && n_frames > 0) {
    codes = ws;
    ws += round_up((size_t)n_frames * kMel, 256);
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int launches = 0;
  cudaError_t e = launch_codes(wav, sample_offsets, frame_offsets, n_clips, n_frames, tails, tails_out, codes, d.err,
                               d.sms, s, &launches);
  if (e == cudaSuccess)
    e = launch_embed(codes, n_frames, table, table_dtype, embed_dim, rms_weight, eps, out, out_dtype, ws, d.err, d.sms,
                     s, &launches, out_rows, out_n_rows, true, G);
  t_last_launches = launches;
  return from_cuda(e);
}
}  // namespace

dmel_status dmel_forward_rows(const float *wav, const int64_t *sample_offsets, const int64_t *frame_offsets,
                              int n_clips, int64_t n_frames, const float *tails, float *tails_out, const void *table,
                              dmel_dtype table_dtype, int embed_dim, const void *rms_weight, float eps, void *out,
                              const int64_t *out_rows, int64_t out_n_rows, dmel_dtype out_dtype, uint8_t *codes_out,
                              void *workspace, size_t workspace_bytes, dmel_stream_t stream) {
  return forward_rows_impl(wav, sample_offsets, frame_offsets, n_clips, n_frames, tails, tails_out, table, table_dtype,
                           embed_dim, rms_weight, eps, nullptr, out, out_rows, out_n_rows, out_dtype, codes_out,
                           workspace, workspace_bytes, stream);
}

dmel_status dmel_forward_prepared(const float *wav, const int64_t *sample_offsets, const int64_t *frame_offsets,
                                  int n_clips, int64_t n_frames, const float *tails, float *tails_out,
                                  const void *table, dmel_dtype table_dtype, int embed_dim, const void *rms_weight,
                                  float eps, const void *prepared, void *out, dmel_dtype out_dtype,
                                  uint8_t *codes_out, void *workspace, size_t workspace_bytes, dmel_stream_t stream) {
  return forward_rows_impl(wav, sample_offsets, frame_offsets, n_clips, n_frames, tails, tails_out, table, table_dtype,
                           embed_dim, rms_weight, eps, prepared, out, nullptr, 0, out_dtype, codes_out, workspace,
                           workspace_bytes, stream);
}

size_t dmel_table_prepare_size(int embed_dim, dmel_dtype table_dtype) {
  // G exists for the tensor-core path's bf16 tables whose width the Gram kernel tiles (128)
  if (table_dtype != DMEL_BF16 || embed_dim <= 0 || embed_dim % 128 != 0) return 0;
  if (!embed_uses_tensor_cores(table_dtype, embed_dim)) return 0;
  return gram_bytes();
}

dmel_status dmel_table_prepare(const void *table, int embed_dim, dmel_dtype table_dtype, void *prepared,
                               size_t prepared_bytes, dmel_stream_t stream) {
  t_last_launches = 0;
  const size_t need = dmel_table_prepare_size(embed_dim, table_dtype);
  if (need == 0 || !table || !aligned(table, 16) || !prepared || !aligned(prepared, 256) || prepared_bytes < need)
    return DMEL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) return DMEL_ERR_CUDA;
  if (d.major != 10) return DMEL_ERR_UNSUPPORTED;
  int launches = 0;
  const cudaError_t e =
      launch_gram(table, embed_dim, static_cast<float *>(prepared), d.err, reinterpret_cast<cudaStream_t>(stream), &launches);
  t_last_launches = launches;
  return from_cuda(e);
}

dmel_status dmel_forward(const float *wav, const int64_t *sample_offsets, const int64_t *frame_offsets, int n_clips,
                         int64_t n_frames, const float *tails, float *tails_out, const void *table,
                         dmel_dtype table_dtype, int embed_dim, const void *rms_weight, float eps, void *out,
                         dmel_dtype out_dtype, uint8_t *codes_out, void *workspace, size_t workspace_bytes,
                         dmel_stream_t stream) {
  return dmel_forward_rows(wav, sample_offsets, frame_offsets, n_clips, n_frames, tails, tails_out, table, table_dtype,
                           embed_dim, rms_weight, eps, out, nullptr, 0, out_dtype, codes_out, workspace,
                           workspace_bytes, stream);
}

namespace {
// Host sample offsets of dmel_forward_host: start 0, non-decreasing.
bool host_offsets_ok(const int64_t *so, int n_clips) {
  if (!so || n_clips < 0 || so[0] != 0) return false;
  for (int c = 0; c < n_clips; ++c)
    if (so[c + 1] < so[c]) return false;
  return true;
}
constexpr int64_t kDefaultChunkFrames = 8192;
}  // namespace

size_t dmel_forward_host_workspace_size(const int64_t *h_sample_offsets, int n_clips, int embed_dim,
                                        dmel_dtype table_dtype, dmel_dtype out_dtype, int with_rmsnorm,
                                        int64_t chunk_frames) {
  if (!host_offsets_ok(h_sample_offsets, n_clips) || embed_dim <= 0 || chunk_frames < 0) return 0;
  if (!dtype_ok(table_dtype) || !dtype_ok(out_dtype)) return 0;
  return forward_host_workspace_bytes(h_sample_offsets, n_clips, embed_dim, table_dtype, out_dtype, with_rmsnorm,
                                      chunk_frames ? chunk_frames : kDefaultChunkFrames);
}

dmel_status dmel_forward_host(const float *h_wav, const int64_t *h_sample_offsets, int n_clips, const void *table,
                              dmel_dtype table_dtype, int embed_dim, const void *rms_weight, float eps, void *h_out,
                              dmel_dtype out_dtype, uint8_t *h_codes, int64_t chunk_frames, void *workspace,
                              size_t workspace_bytes, dmel_stream_t stream) {
  t_last_launches = 0;
  if (!host_offsets_ok(h_sample_offsets, n_clips) || chunk_frames < 0) return DMEL_ERR_INVALID_ARG;
  int64_t F = 0;
  for (int c = 0; c < n_clips; ++c) F += dmel_frames_for_length(h_sample_offsets[c + 1] - h_sample_offsets[c]);
  if (F > 0 && (!h_wav || !h_out)) return DMEL_ERR_INVALID_ARG;
  // the embedding arguments (the codes live in the workspace)
  dmel_status st = check_embed_args(nullptr, false, F, table, table_dtype, embed_dim, rms_weight, eps, h_out,
                                    out_dtype);
  if (st != DMEL_OK || F == 0) return st;
  if (workspace && !aligned(workspace, 256)) return DMEL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) return DMEL_ERR_CUDA;
  if (d.major != 10) return DMEL_ERR_UNSUPPORTED;
  int launches = 0;
  bool too_small = false;
  cudaError_t e = run_forward_host(h_wav, h_sample_offsets, n_clips, table, table_dtype, embed_dim, rms_weight, eps,
                                   h_out, out_dtype, h_codes, chunk_frames ? chunk_frames : kDefaultChunkFrames,
                                   workspace, workspace_bytes, d.err, d.sms, reinterpret_cast<cudaStream_t>(stream),
                                   &launches, &too_small);
  if (too_small) return DMEL_ERR_INVALID_ARG;
  t_last_launches = launches;
  return from_cuda(e);
}

dmel_status dmel_shortconv(const void *x, const int64_t *seq_offsets, int n_seq, int64_t n_tokens, int channels,
                           const float *weights, const void *state, void *state_out, void *y, dmel_dtype dtype,
                           dmel_stream_t stream) {
  t_last_launches = 0;
  if (n_seq < 0 || n_tokens < 0 || channels <= 0 || channels % 8 != 0 || !dtype_ok(dtype)) return DMEL_ERR_INVALID_ARG;
  if (n_seq == 0 && n_tokens > 0) return DMEL_ERR_INVALID_ARG;
  if (n_seq == 0) return DMEL_OK;
  if (!seq_offsets || !weights || !aligned(weights, 16)) return DMEL_ERR_INVALID_ARG;
  if (n_tokens > 0 && (!x || !y || !aligned(x, 16) || !aligned(y, 16))) return DMEL_ERR_INVALID_ARG;
  if ((state && !aligned(state, 16)) || (state_out && !aligned(state_out, 16))) return DMEL_ERR_INVALID_ARG;
  const size_t es = dtype == DMEL_BF16 ? 2 : 4;
  const size_t tok_bytes = (size_t)n_tokens * (size_t)channels * es;
  const size_t st_bytes = (size_t)n_seq * 3 * (size_t)channels * es;
  auto overlap = [](const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return a && b && na && nb && pa < pb + nb && pb < pa + na;
  };
  if (overlap(y, tok_bytes, x, tok_bytes) || overlap(y, tok_bytes, state, st_bytes) ||
      overlap(y, tok_bytes, state_out, st_bytes) || overlap(state_out, st_bytes, x, tok_bytes))
    return DMEL_ERR_INVALID_ARG;
  if (state_out && state && state_out != state && overlap(state_out, st_bytes, state, st_bytes))
    return DMEL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) return DMEL_ERR_CUDA;
  if (d.major != 10) return DMEL_ERR_UNSUPPORTED;
  int launches = 0;
  cudaError_t e = launch_shortconv(x, seq_offsets, n_seq, n_tokens, channels, weights, state, state_out, y, dtype,
                                   d.err, d.sms, reinterpret_cast<cudaStream_t>(stream), &launches);
  t_last_launches = launches;
  return from_cuda(e);
}

namespace {
bool hmlp_weights_ok(const dmel_hmlp_weights *w) {
  if (!w) return false;
  const int dims[4] = {w->d1, w->d2, w->d3, w->dim};
  for (int d : dims)
    if (d <= 0 || d % 8 != 0) return false;
  const void *ptrs[14] = {w->w1, w->w2, w->w3, w->w4, w->b1, w->b2, w->b3, w->b4,
                          w->g1, w->g2, w->g3, w->be1, w->be2, w->be3};
  for (const void *p : ptrs)
    if (!p || !aligned(p, 16)) return false;
  return true;
}
}  // namespace

size_t dmel_hmlp_workspace_size(int64_t n_patches, const dmel_hmlp_weights *w) {
  if (n_patches <= 0 || !hmlp_weights_ok(w)) return 0;
  return hmlp_workspace_bytes(n_patches, *w);
}

dmel_status dmel_hmlp(const void *images, int n_images, int height, int width, const dmel_hmlp_weights *w, void *out,
                      void *workspace, size_t workspace_bytes, dmel_stream_t stream) {
  t_last_launches = 0;
  if (n_images < 0 || height < 0 || width < 0 || height % 40 != 0 || width % 40 != 0) return DMEL_ERR_INVALID_ARG;
  if (!hmlp_weights_ok(w)) return DMEL_ERR_INVALID_ARG;
  const int64_t P = (int64_t)n_images * (height / 40) * (width / 40);
  if (P == 0) return DMEL_OK;
  if (!images || !out || !aligned(images, 16) || !aligned(out, 16)) return DMEL_ERR_INVALID_ARG;
  const size_t need = hmlp_workspace_bytes(P, *w);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return DMEL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) return DMEL_ERR_CUDA;
  if (d.major != 10) return DMEL_ERR_UNSUPPORTED;
  int launches = 0;
  cudaError_t e = launch_hmlp(images, n_images, height, width, *w, out, workspace, d.err, d.sms,
                              reinterpret_cast<cudaStream_t>(stream), &launches);
  t_last_launches = launches;
  return from_cuda(e);
}

dmel_status dmel_splice_plan(const int64_t *h_sentinel_pos, int n_items, const int64_t *h_frame_offsets,
                             int64_t seq_len, int64_t *h_token_pos, int64_t *h_frame_rows,
                             int64_t *h_expanded_len, int64_t *h_audio_tokens) {
  if (seq_len < 0 || n_items < 0 || !h_frame_offsets || (n_items > 0 && !h_sentinel_pos)) return DMEL_ERR_INVALID_ARG;
  if (h_frame_offsets[0] != 0) return DMEL_ERR_INVALID_ARG;
  for (int i = 0; i < n_items; ++i) {
    if (h_sentinel_pos[i] < 0 || h_sentinel_pos[i] >= seq_len) return DMEL_ERR_INVALID_ARG;
    if (i > 0 && h_sentinel_pos[i] <= h_sentinel_pos[i - 1]) return DMEL_ERR_INVALID_ARG;
    if (h_frame_offsets[i + 1] < h_frame_offsets[i]) return DMEL_ERR_INVALID_ARG;
  }
  // walk the original positions once; shift = positions gained so far (sum of f_i - 1)
  int64_t shift = 0;
  int item = 0;
  for (int64_t p = 0; p < seq_len; ++p) {
    if (item < n_items && p == h_sentinel_pos[item]) {
      const int64_t f0 = h_frame_offsets[item], f = h_frame_offsets[item + 1] - f0;
      if (h_token_pos) h_token_pos[p] = -1;
      if (h_frame_rows)
        for (int64_t j = 0; j < f; ++j) h_frame_rows[f0 + j] = p + shift + j;
      shift += f - 1;
      ++item;
    } else if (h_token_pos) {
      h_token_pos[p] = p + shift;
    }
  }
  if (h_expanded_len) *h_expanded_len = seq_len + shift;
  if (h_audio_tokens) *h_audio_tokens = h_frame_offsets[n_items];
  return DMEL_OK;
}

dmel_status dmel_embed_noalloc(const uint8_t *codes, int64_t n_frames, const void *table, dmel_dtype table_dtype,
                               int embed_dim, const void *rms_weight, float eps, void *out, dmel_dtype out_dtype,
                               dmel_stream_t stream) {
  t_last_launches = 0;
  dmel_status st =
      check_embed_args(codes, true, n_frames, table, table_dtype, embed_dim, rms_weight, eps, out, out_dtype);
  if (st != DMEL_OK || n_frames == 0) return st;
  const size_t need = embed_exchange_workspace_bytes(n_frames, embed_dim, table_dtype, rms_weight != nullptr);
  if (need > kNoAllocScratchBytes) return DMEL_ERR_TOO_LARGE;
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) return DMEL_ERR_CUDA;
  if (d.major != 10) return DMEL_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  if (need > 0 && noalloc_scratch(&scratch) != cudaSuccess) return DMEL_ERR_CUDA;
  int launches = 0;
  cudaError_t e = launch_embed(codes, n_frames, table, table_dtype, embed_dim, rms_weight, eps, out, out_dtype,
                               scratch, d.err, d.sms, reinterpret_cast<cudaStream_t>(stream), &launches, nullptr, 0,
                               false);
  t_last_launches = launches;
  return from_cuda(e);
}

dmel_status dmel_get_device_error(uint32_t *h_bits, int clear) {
  if (!h_bits) return DMEL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) return DMEL_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return DMEL_ERR_CUDA;
  if (cudaMemcpy(h_bits, d.err, sizeof(uint32_t), cudaMemcpyDeviceToHost) != cudaSuccess) return DMEL_ERR_CUDA;
  if (clear && cudaMemset(d.err, 0, sizeof(uint32_t)) != cudaSuccess) return DMEL_ERR_CUDA;
  if (clear && cudaDeviceSynchronize() != cudaSuccess) return DMEL_ERR_CUDA;
  return DMEL_OK;
}

const char *dmel_status_string(dmel_status status) {
  switch (status) {
    case DMEL_OK: return "DMEL_OK";
    case DMEL_ERR_INVALID_ARG: return "DMEL_ERR_INVALID_ARG: argument out of contract";
    case DMEL_ERR_UNSUPPORTED: return "DMEL_ERR_UNSUPPORTED: request not supported on this device";
    case DMEL_ERR_CUDA: return "DMEL_ERR_CUDA: a CUDA call or kernel launch failed";
    case DMEL_ERR_TOO_LARGE: return "DMEL_ERR_TOO_LARGE: request needs more than the fixed 4 MiB scratch";
  }
  return "DMEL_ERR_UNKNOWN";
}

int dmel_last_launch_count(void) { return t_last_launches; }

dmel_status dmel_debug_wait_timeout(uint32_t polls, uint32_t *h_bits) {
  if (!h_bits || polls == 0) return DMEL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) return DMEL_ERR_CUDA;
  if (d.major != 10) return DMEL_ERR_UNSUPPORTED;
  int returned = 0;
  if (run_wait_timeout_selftest(polls, d.err, &returned) != cudaSuccess || returned != 1) return DMEL_ERR_CUDA;
  return dmel_get_device_error(h_bits, 1);
}

dmel_status dmel_debug_codes_frame_host_q(const float *frame1600, const dmel_quantizer *q, uint8_t *codes80,
                                          double *lhat80) {
  Quant qz;
  if (!frame1600 || !codes80 || !to_quant(q, &qz)) return DMEL_ERR_INVALID_ARG;
  emulate_codes_frame_host(frame1600, codes80, lhat80, qz);
  return DMEL_OK;
}

dmel_status dmel_debug_forward_host_plan(const int64_t *h_sample_offsets, int n_clips, int64_t chunk_frames,
                                         int64_t *h_plan, int64_t cap, int64_t *h_len) {
  if (!host_offsets_ok(h_sample_offsets, n_clips) || chunk_frames <= 0 || !h_len || cap < 0 || (cap > 0 && !h_plan))
    return DMEL_ERR_INVALID_ARG;
  *h_len = debug_forward_host_plan(h_sample_offsets, n_clips, chunk_frames, h_plan, cap);
  return DMEL_OK;
}

dmel_status dmel_debug_gram(const void *table, int embed_dim, float *gram, dmel_stream_t stream) {
  t_last_launches = 0;
  if (!table || !gram || embed_dim <= 0 || embed_dim % 128 != 0 || !aligned(table, 16) || !aligned(gram, 256))
    return DMEL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) return DMEL_ERR_CUDA;
  if (d.major != 10) return DMEL_ERR_UNSUPPORTED;
  int launches = 0;
  cudaError_t e = launch_gram(table, embed_dim, gram, d.err, reinterpret_cast<cudaStream_t>(stream), &launches);
  t_last_launches = launches;
  return from_cuda(e);
}

dmel_status dmel_debug_norm_sumsq_host(const uint8_t *codes80, const float *h_gram, double *h_sumsq) {
  if (!codes80 || !h_gram || !h_sumsq) return DMEL_ERR_INVALID_ARG;
  for (int b = 0; b < kMel; ++b)
    if (codes80[b] > 15) return DMEL_ERR_INVALID_ARG;
  *h_sumsq = norm_sumsq_host(codes80, h_gram);
  return DMEL_OK;
}

dmel_status dmel_debug_gemm(const void *a, int64_t m, int k, int lda, const void *b, int n, float *c,
                            dmel_stream_t stream) {
  t_last_launches = 0;
  if (m < 0 || m > (int64_t)INT32_MAX || k <= 0 || n <= 0 || lda < k || k % 8 || n % 8 || lda % 8)
    return DMEL_ERR_INVALID_ARG;
  if (m == 0) return DMEL_OK;
  if (!a || !b || !c || !aligned(a, 16) || !aligned(b, 16) || !aligned(c, 16)) return DMEL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) return DMEL_ERR_CUDA;
  if (d.major != 10) return DMEL_ERR_UNSUPPORTED;
  const cudaError_t e = launch_gemm_debug(a, m, k, lda, b, n, c, d.err, d.sms, reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) t_last_launches = 1;
  return from_cuda(e);
}

dmel_status dmel_debug_gelu(const float *x, float *y, int64_t n, dmel_stream_t stream) {
  t_last_launches = 0;
  if (n < 0) return DMEL_ERR_INVALID_ARG;
  if (n == 0) return DMEL_OK;
  if (!x || !y || !aligned(x, 16) || !aligned(y, 16)) return DMEL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (device_info(&d) != cudaSuccess) return DMEL_ERR_CUDA;
  if (d.major != 10) return DMEL_ERR_UNSUPPORTED;
  t_last_launches = 1;
  return from_cuda(launch_gelu_debug(x, y, n, d.sms, reinterpret_cast<cudaStream_t>(stream)));
}

void dmel_debug_codes_frame_host(const float *frame1600, uint8_t *codes80, double *lhat80) {
  emulate_codes_frame_host(frame1600, codes80, lhat80);
}

}  // extern "C"
