// The hierarchical MLP patchifier of the vision path ("Inside Inkling: Audio Design", Part 1 ·
// Modeling: a 4-layer hMLP over 40x40 patches; "Why Thinking Machines Built Inkling Without a
// Vision Encoder": linear layers progressively merge pixels into one embedding per patch).
// Stage 1 maps every 5x5 pixel block (75 values, row / column / channel order) to d1 features;
// stages 2-4 map every 2x2 group of the previous stage's grid (four vectors concatenated in
// top-left, top-right, bottom-left, bottom-right order) to d2, d3 and finally dim features.
// Bias, LayerNorm (eps 1e-6) and the exact GELU follow stages 1-3, bias alone stage 4; every
// stage's output is stored in bf16.
//
// Within a patch the blocks are kept in Morton (quad-tree) order, so the four children of a
// 2x2 group are four consecutive rows and every merge is the previous stage's output read as
// [rows / 4 x 4 d]: no data moves between stages. The four products are plain dense GEMMs
// (cuBLASLt, bf16 x bf16 -> fp32); the pixel gather and the fused bias / LayerNorm / GELU /
// rounding run in this file's kernels.
#include <cublasLt.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dmel {
namespace {

constexpr int kPatch = 40;
constexpr int kBlocks = 64;   // 5x5 blocks per patch (8 x 8)
constexpr int kK1 = 75;       // values per block
constexpr int kK1Pad = 80;    // row stride of the gathered blocks (16-byte rows)
constexpr size_t kLtWorkspace = size_t(32) << 20;

__host__ __device__ inline int demorton_r(int m) { return ((m >> 1) & 1) | ((m >> 2) & 2) | ((m >> 3) & 4); }
__host__ __device__ inline int demorton_c(int m) { return (m & 1) | ((m >> 1) & 2) | ((m >> 2) & 4); }

// One thread per (patch, block): the block's 75 pixel values, then 5 zeros, as one bf16 row.
__global__ void __launch_bounds__(256) hmlp_gather_kernel(const __nv_bfloat16 *__restrict__ img, int n, int H, int W,
                                                          __nv_bfloat16 *__restrict__ A) {
  const int pw = W / kPatch, ph = H / kPatch;
  const int64_t total = (int64_t)n * ph * pw * kBlocks;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t p = idx / kBlocks;
    const int m = (int)(idx % kBlocks);
    const int i = (int)(p / ((int64_t)ph * pw));
    const int pr = (int)((p / pw) % ph), pc = (int)(p % pw);
    const int r0 = kPatch * pr + 5 * demorton_r(m), c0 = kPatch * pc + 5 * demorton_c(m);
    __nv_bfloat16 *out = A + idx * kK1Pad;
    for (int kr = 0; kr < 5; ++kr) {
      const __nv_bfloat16 *src = img + (((int64_t)i * H + r0 + kr) * W + c0) * 3;
      for (int q = 0; q < 15; ++q) out[kr * 15 + q] = src[q];
    }
    for (int q = kK1; q < kK1Pad; ++q) out[q] = __float2bfloat16_rn(0.0f);
  }
}

// One warp per row of d fp32 sums: + bias, then (kNorm) LayerNorm with gain / shift and the
// exact GELU, rounded to bf16. Mean first, then the mean squared deviation (two passes).
template <bool kNorm>
__global__ void __launch_bounds__(256) hmlp_row_kernel(const float *__restrict__ in, int64_t rows, int d,
                                                       const float *__restrict__ bias, const float *__restrict__ g,
                                                       const float *__restrict__ be, __nv_bfloat16 *__restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const float *x = in + r * d;
    __nv_bfloat16 *y = out + r * d;
    float mean = 0.0f, rstd = 1.0f;
    if (kNorm) {
      float s = 0.0f;
      for (int j = 4 * lane; j < d; j += 128) {
        const float4 v = *reinterpret_cast<const float4 *>(x + j), b = *reinterpret_cast<const float4 *>(bias + j);
        s += (v.x + b.x) + (v.y + b.y) + (v.z + b.z) + (v.w + b.w);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      mean = s / (float)d;
      float q = 0.0f;
      for (int j = 4 * lane; j < d; j += 128) {
        const float4 v = *reinterpret_cast<const float4 *>(x + j), b = *reinterpret_cast<const float4 *>(bias + j);
        const float e0 = v.x + b.x - mean, e1 = v.y + b.y - mean, e2 = v.z + b.z - mean, e3 = v.w + b.w - mean;
        q += e0 * e0 + e1 * e1 + e2 * e2 + e3 * e3;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
      rstd = 1.0f / sqrtf(q / (float)d + 1e-6f);
    }
    for (int j = 4 * lane; j < d; j += 128) {
      const float4 v = *reinterpret_cast<const float4 *>(x + j), b = *reinterpret_cast<const float4 *>(bias + j);
      float t[4] = {v.x + b.x, v.y + b.y, v.z + b.z, v.w + b.w};
      if (kNorm) {
        const float4 gg = *reinterpret_cast<const float4 *>(g + j), bb = *reinterpret_cast<const float4 *>(be + j);
        const float gv[4] = {gg.x, gg.y, gg.z, gg.w}, bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float u = (t[k] - mean) * rstd * gv[k] + bv[k];
          t[k] = 0.5f * u * (1.0f + erff(u * 0.70710678118654752f));
        }
      }
      __nv_bfloat162 lo = __floats2bfloat162_rn(t[0], t[1]), hi = __floats2bfloat162_rn(t[2], t[3]);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t *>(&lo);
      pk.y = *reinterpret_cast<uint32_t *>(&hi);
      *reinterpret_cast<uint2 *>(y + j) = pk;
    }
  }
}

// cuBLASLt handle per device (created on first use, kept for the process).
std::mutex g_lt_mu;
cublasLtHandle_t g_lt[256] = {nullptr};

cudaError_t lt_handle(cublasLtHandle_t *h) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_lt_mu);
  if (!g_lt[dev & 255] && cublasLtCreate(&g_lt[dev & 255]) != CUBLAS_STATUS_SUCCESS) return cudaErrorUnknown;
  *h = g_lt[dev & 255];
  return cudaSuccess;
}

// Row-major C [M x N] fp32 = A [M x K] (row stride lda) * B [K x N], bf16 inputs, fp32 sums:
// column-major C^T = B^T A^T for cuBLASLt.
cudaError_t lt_gemm(cublasLtHandle_t h, const __nv_bfloat16 *A, int64_t M, int K, int lda, const __nv_bfloat16 *B,
                    int N, float *C, void *ws, cudaStream_t stream) {
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  cudaError_t result = cudaErrorUnknown;
  do {
    if (cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS) break;
    // the column-major operands: first B^T [N x K] (ld N), second A^T [K x M] (ld lda)
    if (cublasLtMatrixLayoutCreate(&lb, CUDA_R_16BF, N, K, N) != CUBLAS_STATUS_SUCCESS) break;
    if (cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, K, M, lda) != CUBLAS_STATUS_SUCCESS) break;
    if (cublasLtMatrixLayoutCreate(&lc, CUDA_R_32F, N, M, N) != CUBLAS_STATUS_SUCCESS) break;
    if (cublasLtMatmulPreferenceCreate(&pref) != CUBLAS_STATUS_SUCCESS) break;
    size_t wsb = kLtWorkspace;
    if (cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &wsb, sizeof(wsb)) !=
        CUBLAS_STATUS_SUCCESS)
      break;
    cublasLtMatmulHeuristicResult_t heur;
    int found = 0;
    if (cublasLtMatmulAlgoGetHeuristic(h, op, lb, la, lc, lc, pref, 1, &heur, &found) != CUBLAS_STATUS_SUCCESS ||
        found < 1)
      break;
    const float alpha = 1.0f, beta = 0.0f;
    if (cublasLtMatmul(h, op, &alpha, B, lb, A, la, &beta, C, lc, C, lc, &heur.algo, ws, kLtWorkspace, stream) !=
        CUBLAS_STATUS_SUCCESS)
      break;
    result = cudaGetLastError();
  } while (false);
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (la) cublasLtMatrixLayoutDestroy(la);
  if (lb) cublasLtMatrixLayoutDestroy(lb);
  if (op) cublasLtMatmulDescDestroy(op);
  return result;
}

size_t r256(size_t x) { return (x + 255) / 256 * 256; }

struct HmlpLayout {
  size_t a1, h13, h2, f32, lt, total;
};

HmlpLayout hmlp_layout(int64_t P, const dmel_hmlp_weights &w) {
  const size_t rows1 = (size_t)P * kBlocks, rows2 = (size_t)P * 16, rows3 = (size_t)P * 4;
  HmlpLayout L;
  L.a1 = r256(rows1 * kK1Pad * 2);
  const size_t h1 = rows1 * (size_t)w.d1, h3 = rows3 * (size_t)w.d3;
  L.h13 = r256((h1 > h3 ? h1 : h3) * 2);
  L.h2 = r256(rows2 * (size_t)w.d2 * 2);
  size_t f = rows1 * (size_t)w.d1;
  if (rows2 * (size_t)w.d2 > f) f = rows2 * (size_t)w.d2;
  if (rows3 * (size_t)w.d3 > f) f = rows3 * (size_t)w.d3;
  if ((size_t)P * (size_t)w.dim > f) f = (size_t)P * (size_t)w.dim;
  L.f32 = r256(f * 4);
  L.lt = kLtWorkspace;
  L.total = L.a1 + L.h13 + L.h2 + L.f32 + L.lt;
  return L;
}

template <bool kNorm>
cudaError_t launch_rows(const float *in, int64_t rows, int d, const float *b, const float *g, const float *be,
                        __nv_bfloat16 *out, int num_sms, cudaStream_t stream) {
  const int64_t blocks = (rows + 7) / 8;
  const int64_t cap = (int64_t)num_sms * 16;
  hmlp_row_kernel<kNorm><<<(unsigned)(blocks < cap ? blocks : cap), 256, 0, stream>>>(in, rows, d, b, g, be, out);
  return cudaGetLastError();
}

}  // namespace

size_t hmlp_workspace_bytes(int64_t n_patches, const dmel_hmlp_weights &w) {
  return n_patches > 0 ? hmlp_layout(n_patches, w).total : 0;
}

cudaError_t launch_hmlp(const void *images, int n, int H, int W, const dmel_hmlp_weights &w, void *out,
                        void *workspace, int num_sms, cudaStream_t stream, int *launches) {
  const int64_t P = (int64_t)n * (H / kPatch) * (W / kPatch);
  if (P <= 0) return cudaSuccess;
  cublasLtHandle_t h;
  cudaError_t e = lt_handle(&h);
  if (e != cudaSuccess) return e;
  const HmlpLayout L = hmlp_layout(P, w);
  uint8_t *base = static_cast<uint8_t *>(workspace);
  auto *A1 = reinterpret_cast<__nv_bfloat16 *>(base);
  auto *H13 = reinterpret_cast<__nv_bfloat16 *>(base + L.a1);
  auto *H2 = reinterpret_cast<__nv_bfloat16 *>(base + L.a1 + L.h13);
  auto *F = reinterpret_cast<float *>(base + L.a1 + L.h13 + L.h2);
  void *lt_ws = base + L.a1 + L.h13 + L.h2 + L.f32;
  const auto *W1 = static_cast<const __nv_bfloat16 *>(w.w1);
  const auto *W2 = static_cast<const __nv_bfloat16 *>(w.w2);
  const auto *W3 = static_cast<const __nv_bfloat16 *>(w.w3);
  const auto *W4 = static_cast<const __nv_bfloat16 *>(w.w4);
  {
    const int64_t items = P * kBlocks;
    const int64_t cap = (int64_t)num_sms * 16;
    const int64_t blocks = (items + 255) / 256;
    hmlp_gather_kernel<<<(unsigned)(blocks < cap ? blocks : cap), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(images), n, H, W, A1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ++*launches;
  }
  const int64_t rows1 = P * kBlocks, rows2 = P * 16, rows3 = P * 4;
  if ((e = lt_gemm(h, A1, rows1, kK1, kK1Pad, W1, w.d1, F, lt_ws, stream)) != cudaSuccess) return e;
  if ((e = launch_rows<true>(F, rows1, w.d1, w.b1, w.g1, w.be1, H13, num_sms, stream)) != cudaSuccess) return e;
  if ((e = lt_gemm(h, H13, rows2, 4 * w.d1, 4 * w.d1, W2, w.d2, F, lt_ws, stream)) != cudaSuccess) return e;
  if ((e = launch_rows<true>(F, rows2, w.d2, w.b2, w.g2, w.be2, H2, num_sms, stream)) != cudaSuccess) return e;
  if ((e = lt_gemm(h, H2, rows3, 4 * w.d2, 4 * w.d2, W3, w.d3, F, lt_ws, stream)) != cudaSuccess) return e;
  if ((e = launch_rows<true>(F, rows3, w.d3, w.b3, w.g3, w.be3, H13, num_sms, stream)) != cudaSuccess) return e;
  if ((e = lt_gemm(h, H13, P, 4 * w.d3, 4 * w.d3, W4, w.dim, F, lt_ws, stream)) != cudaSuccess) return e;
  if ((e = launch_rows<false>(F, P, w.dim, w.b4, nullptr, nullptr, static_cast<__nv_bfloat16 *>(out), num_sms,
                              stream)) != cudaSuccess)
    return e;
  *launches += 4;  // the four row kernels (the four GEMMs are cuBLASLt's)
  return cudaSuccess;
}

}  // namespace dmel
