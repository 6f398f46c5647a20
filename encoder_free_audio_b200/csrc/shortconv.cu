// ShortConv: the per-channel causal convolution of width 4 that the decoder applies after its
// key/value projections and on its residual-branch outputs ("Inside Inkling: Audio Design",
// Part 3 · Inference):  y[t, c] = x[t, c] + sum_{d=0}^{3} w[c, d] x[t - d, c], per sequence, with
// the three inputs before a sequence's first token taken from its carried state.
//
// The operation moves 2 values per output and does 5 multiply-adds: HBM bound. Each thread owns
// 8 channels (one 16-byte bf16 vector, or two fp32 ones) of a run of 32 consecutive tokens and
// slides down it with the last three inputs in registers, so every input is read from memory
// once (plus three history rows at the run's start); consecutive threads own consecutive channel
// groups, so a warp reads and writes whole 512-byte (bf16) row pieces. Each thread keeps its next
// eight tokens in flight with cp.async copies into its own shared-memory slots, which keeps
// enough bytes in flight per SM without holding them in registers.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace dmel {
namespace {

constexpr int kScRun = 32;       // tokens per thread
constexpr int kScThreads = 256;
constexpr int kScDepth = 8;      // tokens each thread keeps in flight (cp.async into shared memory)

__device__ __forceinline__ void cp_async16(uint32_t smem_dst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_dst), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// 8 channels of one token from this thread's staging slot (written by its own cp.async).
__device__ __forceinline__ void sc_smem8(const uint8_t *p, const float *, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 16);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void sc_smem8(const uint8_t *p, const __nv_bfloat16 *, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4 *>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ void sc_load8(const float *p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4 *>(p)), b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void sc_load8(const __nv_bfloat16 *p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ void sc_store8(float *p, const float (&v)[8]) {
  __stcs(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
  __stcs(reinterpret_cast<float4 *>(p) + 1, make_float4(v[4], v[5], v[6], v[7]));
}

__device__ __forceinline__ void sc_store8(__nv_bfloat16 *p, const float (&v)[8]) {
  uint4 u;
  __nv_bfloat162 h;
  h = __floats2bfloat162_rn(v[0], v[1]); u.x = *reinterpret_cast<uint32_t *>(&h);
  h = __floats2bfloat162_rn(v[2], v[3]); u.y = *reinterpret_cast<uint32_t *>(&h);
  h = __floats2bfloat162_rn(v[4], v[5]); u.z = *reinterpret_cast<uint32_t *>(&h);
  h = __floats2bfloat162_rn(v[6], v[7]); u.w = *reinterpret_cast<uint32_t *>(&h);
  __stcs(reinterpret_cast<uint4 *>(p), u);
}

// Input at position j (relative to the start of sequence s, j < 0 reaching into the carried
// state) for channel group g; zeros without a state. Positions outside the token range (bad
// offsets) read as zero and are recorded.
template <typename T>
__device__ __forceinline__ void sc_fetch(const T *x, const T *state, const int64_t *off, int s, int64_t j, int C,
                                         int g, int64_t n_tok, uint32_t *err, float (&v)[8]) {
  if (j >= 0) {
    const int64_t t = off[s] + j;
    if (t >= 0 && t < n_tok) {
      sc_load8(x + t * (int64_t)C + 8 * g, v);
      return;
    }
    record_error(err, DMEL_DEVERR_OFFSETS);
  } else if (state && j >= -3) {
    sc_load8(state + ((int64_t)s * 3 + 3 + j) * C + 8 * g, v);
    return;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = 0.0f;
}

template <typename T>
__global__ void __launch_bounds__(kScThreads, 3) shortconv_kernel(const T *__restrict__ x, const int64_t *__restrict__ off,
                                                               int n_seq, int64_t n_tok, int C,
                                                               const float *__restrict__ w, const T *state,
                                                               T *__restrict__ y, uint32_t *err) {
  extern __shared__ __align__(16) uint8_t sc_stage[];
  constexpr int kPieces = (int)sizeof(T) / 2;  // 16-byte pieces per 8 channels: 1 (bf16), 2 (fp32)
  const uint32_t slot_stride = (uint32_t)(blockDim.x * 16 * kPieces);
  const uint8_t *stage_ptr = sc_stage + threadIdx.x * 16 * kPieces;
  const uint32_t stage = smem_addr(stage_ptr);
  const int G = C / 8;
  const int64_t runs = (n_tok + kScRun - 1) / kScRun;
  const int64_t items = runs * G;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items; it += (int64_t)gridDim.x * blockDim.x) {
    const int g = (int)(it % G);
    const int64_t t0 = (it / G) * kScRun;
    const int64_t t1 = t0 + kScRun < n_tok ? t0 + kScRun : n_tok;
    // sequence holding t0: the last s with off[s] <= t0
    int lo = 0, hi = n_seq - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (off[mid] <= t0) lo = mid; else hi = mid - 1;
    }
    int s = lo;
    float wt[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 q = __ldg(reinterpret_cast<const float4 *>(w + (int64_t)(8 * g + i) * 4));
      wt[i][0] = q.x; wt[i][1] = q.y; wt[i][2] = q.z; wt[i][3] = q.w;
    }
    float h1[8], h2[8], h3[8];
    int64_t j0 = t0 - off[s];  // position of t0 in its sequence
    sc_fetch(x, state, off, s, j0 - 1, C, g, n_tok, err, h1);
    sc_fetch(x, state, off, s, j0 - 2, C, g, n_tok, err, h2);
    sc_fetch(x, state, off, s, j0 - 3, C, g, n_tok, err, h3);
    // one output from the current input and history, then the history shifts by one token
    auto step = [&](const float (&xt)[8], float (&yt)[8]) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float acc = xt[i];
        acc = fmaf(wt[i][0], xt[i], acc);
        acc = fmaf(wt[i][1], h1[i], acc);
        acc = fmaf(wt[i][2], h2[i], acc);
        acc = fmaf(wt[i][3], h3[i], acc);
        yt[i] = acc;
        h3[i] = h2[i];
        h2[i] = h1[i];
        h1[i] = xt[i];
      }
    };
    // this thread's tokens t0 .. t1 - 1 stream through kScDepth staging slots (slot k at
    // stage + k * slot_stride); one commit group per token, empty past t1
    auto issue = [&](int64_t tt, int k) {
      if (tt < t1) {
        const T *src = x + tt * (int64_t)C + 8 * g;
#pragma unroll
        for (int q = 0; q < kPieces; ++q) cp_async16(stage + k * slot_stride + 16 * q, reinterpret_cast<const uint8_t *>(src) + 16 * q);
      }
      cp_async_commit();
    };
#pragma unroll
    for (int k = 0; k < kScDepth; ++k) issue(t0 + k, k);
    for (int64_t t = t0; t < t1; ++t) {
      if (s + 1 < n_seq && t >= off[s + 1]) {  // a new sequence starts at t (empty ones skipped)
        while (s + 1 < n_seq && t >= off[s + 1]) ++s;
        sc_fetch(x, state, off, s, -1, C, g, n_tok, err, h1);
        sc_fetch(x, state, off, s, -2, C, g, n_tok, err, h2);
        sc_fetch(x, state, off, s, -3, C, g, n_tok, err, h3);
      }
      const int k = (int)((t - t0) % kScDepth);
      cp_async_wait<kScDepth - 1>();  // the group of token t has landed
      float xt[8], yt[8];
      sc_smem8(stage_ptr + k * slot_stride, x, xt);
      issue(t + kScDepth, k);  // the slot is free again: token t + depth into it
      step(xt, yt);
      sc_store8(y + t * (int64_t)C + 8 * g, yt);
    }
    cp_async_wait<0>();
  }
}

// Carried state out: the last three inputs of each sequence (from the state in where the
// sequence is shorter). One thread per (sequence, channel group) reads its three rows before
// writing any, so state_out may be the state in.
template <typename T>
__global__ void __launch_bounds__(kScThreads) shortconv_state_kernel(const T *__restrict__ x, const int64_t *off,
                                                                     int n_seq, int64_t n_tok, int C, const T *state,
                                                                     T *state_out, uint32_t *err) {
  const int G = C / 8;
  const int64_t items = (int64_t)n_seq * G;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items; it += (int64_t)gridDim.x * blockDim.x) {
    const int g = (int)(it % G);
    const int s = (int)(it / G);
    const int64_t len = off[s + 1] - off[s];
    float v[3][8];
#pragma unroll
    for (int i = 0; i < 3; ++i) sc_fetch(x, state, off, s, len - 3 + i, C, g, n_tok, err, v[i]);
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      T *dst = state_out + ((int64_t)s * 3 + i) * C + 8 * g;
      float o[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = v[i][k];
      if (sizeof(T) == 4) {
        reinterpret_cast<float4 *>(dst)[0] = make_float4(o[0], o[1], o[2], o[3]);
        reinterpret_cast<float4 *>(dst)[1] = make_float4(o[4], o[5], o[6], o[7]);
      } else {
        sc_store8(dst, o);
      }
    }
  }
}

template <typename T>
cudaError_t launch_sc(const T *x, const int64_t *off, int n_seq, int64_t n_tok, int C, const float *w, const T *state,
                      T *state_out, T *y, uint32_t *err, int num_sms, cudaStream_t stream, int *launches) {
  const int64_t G = C / 8;
  if (n_tok > 0) {
    const int64_t items = ((n_tok + kScRun - 1) / kScRun) * G;
    const int64_t cap = (int64_t)num_sms * 8;
    const int64_t blocks = (items + kScThreads - 1) / kScThreads;
    const int smem = kScDepth * kScThreads * 16 * ((int)sizeof(T) / 2);
    static std::atomic<bool> attr[256];
    const cudaError_t e0 = set_smem_attr_once(shortconv_kernel<T>, smem, attr);
    if (e0 != cudaSuccess) return e0;
    shortconv_kernel<T><<<(unsigned)(blocks < cap ? blocks : cap), kScThreads, smem, stream>>>(x, off, n_seq, n_tok, C,
                                                                                             w, state, y, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  if (state_out && n_seq > 0) {
    const int64_t items = (int64_t)n_seq * G;
    const int64_t cap = (int64_t)num_sms * 8;
    const int64_t blocks = (items + kScThreads - 1) / kScThreads;
    shortconv_state_kernel<T><<<(unsigned)(blocks < cap ? blocks : cap), kScThreads, 0, stream>>>(
        x, off, n_seq, n_tok, C, state, state_out, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_shortconv(const void *x, const int64_t *seq_offsets, int n_seq, int64_t n_tokens, int channels,
                             const float *weights, const void *state, void *state_out, void *y, dmel_dtype dtype,
                             uint32_t *err, int num_sms, cudaStream_t stream, int *launches) {
  if (dtype == DMEL_BF16)
    return launch_sc(static_cast<const __nv_bfloat16 *>(x), seq_offsets, n_seq, n_tokens, channels, weights,
                     static_cast<const __nv_bfloat16 *>(state), static_cast<__nv_bfloat16 *>(state_out),
                     static_cast<__nv_bfloat16 *>(y), err, num_sms, stream, launches);
  return launch_sc(static_cast<const float *>(x), seq_offsets, n_seq, n_tokens, channels, weights,
                   static_cast<const float *>(state), static_cast<float *>(state_out), static_cast<float *>(y), err,
                   num_sms, stream, launches);
}

}  // namespace dmel
