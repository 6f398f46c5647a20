// ShortConv: the per-channel causal convolution of width 4 that the decoder applies after its
// key/value projections and on its residual-branch outputs ("Inside Inkling: Audio Design",
// Part 3 · Inference):  y[t, c] = x[t, c] + sum_{d=0}^{3} w[c, d] x[t - d, c], per sequence, with
// the three inputs before a sequence's first token taken from its carried state.
//
// The operation moves 2 values per output and does 5 multiply-adds: HBM bound. A block owns a
// slice of up to 2048 channels of a run of consecutive tokens. One producer thread streams the
// slice's rows (4 KB contiguous in bf16) into a ring of shared-memory slots with bulk copies,
// keeping up to 16 rows in flight per block; 256 consumer threads each own 8 channels, keep the
// last three inputs in registers, read each row once from its slot and write the outputs straight
// to global memory (a warp writes 512 contiguous bytes per row). Every input is read from memory
// once, plus three history rows per run. Where the carried state out is a separate buffer, the
// block whose run holds a sequence's last token also writes that sequence's state; otherwise a
// second kernel writes it after the first has read every state in.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace dmel {
namespace {

namespace scv {
constexpr int CW = 2048;                 // channels per block slice
constexpr int SLOTS = 16;                // rows in flight per block
constexpr int CONSUMERS = CW / 8;        // one thread per 8 channels
constexpr int THREADS = CONSUMERS + 32;  // + the producer warp
}  // namespace scv

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from global memory into
// this block's shared memory, completion counted on an mbarrier (no multicast).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// 8 channels of one token from a shared-memory row slot.
__device__ __forceinline__ void sc_slot8(const uint8_t *p, const float *, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 16);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void sc_slot8(const uint8_t *p, const __nv_bfloat16 *, float (&v)[8]) {
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
  reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

__device__ __forceinline__ void sc_store8(__nv_bfloat16 *p, const float (&v)[8]) {
  uint4 u;
  __nv_bfloat162 h;
  h = __floats2bfloat162_rn(v[0], v[1]); u.x = *reinterpret_cast<uint32_t *>(&h);
  h = __floats2bfloat162_rn(v[2], v[3]); u.y = *reinterpret_cast<uint32_t *>(&h);
  h = __floats2bfloat162_rn(v[4], v[5]); u.z = *reinterpret_cast<uint32_t *>(&h);
  h = __floats2bfloat162_rn(v[6], v[7]); u.w = *reinterpret_cast<uint32_t *>(&h);
  *reinterpret_cast<uint4 *>(p) = u;
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

// The sequence holding token t (the last s with off[s] <= t; offsets non-decreasing), found by
// the whole warp: each round the 32 lanes probe 32 evenly spaced points of the remaining range,
// so n sequences take about log32(n) dependent loads instead of log2(n).
__device__ __forceinline__ int sc_find_seq(const int64_t *off, int n_seq, int64_t t, int lane) {
  int lo = 0, hi = n_seq - 1;  // the answer lies in [lo, hi]
  while (hi > lo) {
    const int64_t span = hi - lo;
    const int probe = lo + 1 + (int)((span * lane) / 32);  // in (lo, hi], non-decreasing in lane
    const unsigned le = __ballot_sync(0xffffffffu, off[probe] <= t);
    if (le == 0) {
      hi = lo;  // even the first probe is past t: the answer is lo
    } else {
      const int top = 31 - __clz(le);  // the last probe at or before t
      const int nlo = lo + 1 + (int)((span * top) / 32);
      const int nhi = top == 31 ? hi : lo + 1 + (int)((span * (top + 1)) / 32) - 1;
      lo = nlo;
      hi = nhi;
    }
  }
  return lo;
}

template <typename T>
__global__ void __launch_bounds__(scv::THREADS, 2) shortconv_kernel(const T *__restrict__ x, const int64_t *__restrict__ off,
                                                                 int n_seq, int64_t n_tok, int C,
                                                                 const float *__restrict__ w, const T *state,
                                                                 T *__restrict__ y, T *state_out, int n_slices,
                                                                 int64_t run_len, uint32_t *err) {
  using namespace scv;
  extern __shared__ __align__(128) uint8_t sc_smem[];
  constexpr uint32_t kSlot = CW * (uint32_t)sizeof(T);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slice = (int)(blockIdx.x % n_slices);
  const int64_t t0 = (int64_t)(blockIdx.x / n_slices) * run_len;
  const int64_t t1 = t0 + run_len < n_tok ? t0 + run_len : n_tok;
  const int c0 = slice * CW;
  const int cw = C - c0 < CW ? C - c0 : CW;
  const uint32_t row_bytes = (uint32_t)cw * (uint32_t)sizeof(T);
  const uint32_t bar0 = smem_addr(sc_smem + SLOTS * kSlot);
  auto full = [&](int k) { return bar0 + 8u * k; };
  auto empty = [&](int k) { return bar0 + 8u * (SLOTS + k); };
  if (threadIdx.x == 0) {
    for (int k = 0; k < SLOTS; ++k) {
      mbar_init(full(k), 1);
      mbar_init(empty(k), CONSUMERS / 32);
    }
    mbar_fence_init();
  }
  __syncthreads();
  if (t0 >= t1) return;

  if (warp == CONSUMERS / 32) {
    // ------------------------------------------------ producer: rows t0 .. t1 - 1 into the ring
    if (lane == 0) {
      int64_t n = 0;
      int k = 0;
      uint32_t ph = 0;
      for (int64_t t = t0; t < t1; ++t, ++n) {
        // from the second round on, the slot's previous row has been read by every warp
        if (n >= SLOTS && !mbar_wait(empty(k), ph ^ 1u, err)) break;
        mbar_arrive_expect_tx(full(k), row_bytes);
        bulk_load(smem_addr(sc_smem + k * kSlot), x + t * (int64_t)C + c0, row_bytes, full(k));
        if (++k == SLOTS) { k = 0; ph ^= 1u; }
      }
      // every copy this thread started has landed before the block's shared memory goes away
      for (int64_t q = n > SLOTS ? n - SLOTS : 0; q < n; ++q)
        mbar_wait(full((int)(q % SLOTS)), (uint32_t)(q / SLOTS) & 1u, err);
    }
    return;
  }

  // ------------------------------------------------ consumers: 8 channels of every row
  const int g = threadIdx.x;  // channel group within the slice
  const bool active = 8 * g < cw;
  const int ch = c0 + 8 * g;
  int s = sc_find_seq(off, n_seq, t0, lane);
  int64_t next_start = s + 1 < n_seq ? off[s + 1] : INT64_MAX;
  float wt[8][4];
  const int gg = active ? ch / 8 : 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 q = __ldg(reinterpret_cast<const float4 *>(w + (int64_t)(8 * gg + i) * 4));
    wt[i][0] = q.x; wt[i][1] = q.y; wt[i][2] = q.z; wt[i][3] = q.w;
  }
  float h1[8], h2[8], h3[8];  // the inputs one, two and three tokens back
  {
    const int64_t j0 = t0 - off[s];  // position of t0 in its sequence
    sc_fetch(x, state, off, s, j0 - 1, C, gg, n_tok, err, h1);
    sc_fetch(x, state, off, s, j0 - 2, C, gg, n_tok, err, h2);
    sc_fetch(x, state, off, s, j0 - 3, C, gg, n_tok, err, h3);
  }
  int k = 0;        // ring slot of the next row
  uint32_t ph = 0;  // its phase
  bool ok = true;
  for (int64_t t = t0; t < t1; ++t) {
    if (t >= next_start) {  // a new sequence starts at t (empty ones skipped): its carried state
      while (s + 1 < n_seq && t >= off[s + 1]) ++s;
      next_start = s + 1 < n_seq ? off[s + 1] : INT64_MAX;
      sc_fetch(x, state, off, s, -1, C, gg, n_tok, err, h1);
      sc_fetch(x, state, off, s, -2, C, gg, n_tok, err, h2);
      sc_fetch(x, state, off, s, -3, C, gg, n_tok, err, h3);
    }
    if (!__all_sync(0xffffffffu, mbar_wait(full(k), ph, err))) { ok = false; break; }
    float xt[8];
    sc_slot8(sc_smem + k * kSlot + 16 * g * (sizeof(T) / 2), x, xt);
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(k));  // the warp's reads of the slot are done
    if (++k == SLOTS) { k = 0; ph ^= 1u; }
    float yt[8];
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
    if (active) sc_store8(y + t * (int64_t)C + ch, yt);
  }
  if (state_out && ok) {
    // carried state out of the sequences that end in this run (token off[q + 1] - 1 in
    // [t0, t1); the first run also takes the empty sequences at offset 0): their last three
    // inputs, or the state in where a sequence is shorter. state_out is not the state in here.
    int q = 0;
    if (t0 > 0) {  // first q with off[q + 1] > t0
      int a = 0, b = n_seq;
      while (a < b) {
        const int mid = (a + b) >> 1;
        if (off[mid + 1] > t0) b = mid; else a = mid + 1;
      }
      q = a;
    }
    // (the last run also takes sequences said to end past the last token: their fetches flag it)
    for (; q < n_seq && (off[q + 1] <= t1 || t1 == n_tok); ++q) {
      const int64_t len = off[q + 1] - off[q];
#pragma unroll 1
      for (int i = 0; i < 3; ++i) {
        float v[8];
        sc_fetch(x, state, off, q, len - 3 + i, C, gg, n_tok, err, v);
        if (active) sc_store8(state_out + ((int64_t)q * 3 + i) * C + ch, v);
      }
    }
  }
}

// Carried state out: the last three inputs of each sequence (from the state in where the
// sequence is shorter). One thread per (sequence, channel group) reads its three rows before
// writing any, so state_out may be the state in.
template <typename T>
__global__ void __launch_bounds__(256) shortconv_state_kernel(const T *__restrict__ x, const int64_t *off,
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
    // slices of 2048 channels x runs of consecutive tokens, one per block, two blocks per SM
    const int n_slices = (int)((C + scv::CW - 1) / scv::CW);
    int64_t n_runs = (int64_t)num_sms * 2 / n_slices;
    if (n_runs < 1) n_runs = 1;
    if (n_runs > n_tok) n_runs = n_tok;
    const int64_t run_len = (n_tok + n_runs - 1) / n_runs;
    n_runs = (n_tok + run_len - 1) / run_len;
    const int smem = scv::SLOTS * scv::CW * (int)sizeof(T) + 2 * scv::SLOTS * 8;
    static std::atomic<bool> attr[256];
    const cudaError_t e0 = set_smem_attr_once(shortconv_kernel<T>, smem, attr);
    if (e0 != cudaSuccess) return e0;
    // the state out is written by this kernel unless it is the state in (which the kernel reads)
    T *so = state_out != state ? state_out : nullptr;
    shortconv_kernel<T><<<(unsigned)(n_runs * n_slices), scv::THREADS, smem, stream>>>(
        x, off, n_seq, n_tok, C, w, state, y, so, n_slices, run_len, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  if (state_out && n_seq > 0 && (n_tok == 0 || state_out == state)) {
    const int64_t items = (int64_t)n_seq * G;
    const int64_t cap = (int64_t)num_sms * 8;
    const int64_t blocks = (items + 255) / 256;
    shortconv_state_kernel<T><<<(unsigned)(blocks < cap ? blocks : cap), 256, 0, stream>>>(
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
