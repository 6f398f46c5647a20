// dMel embedding: x_j = sum_b T[16 b + c_b, j] over the 80 channels of a frame, optional
// RMSNorm y_j = g_j x_j / sqrt(mean_j x_j^2 + eps) ("Inside Inkling: Audio Design",
// Part 1 · Modeling: each (bin, level) pair owns one row, a frame's 80 rows are summed,
// optional RMSNorm).
//
// Tensor-core path (bf16 table, D % 256 == 0). The row sum is the product
// onehot(codes) [frames x 1280] . T [1280 x D]: a dense contraction with K = 1280, run as a
// tcgen05 GEMM with fp32 accumulators in TMEM.
//   tile 128 frames x 256 columns, K in 20 blocks of 64 (4 channels x 16 levels);
//   warp 0      TMA loads of the table block [64 rows x 256 cols] (4 boxes of 64 x 64, 128B
//               swizzle, L2 evict-last: the 15.7 MB table stays in L2);
//   warp 1      allocates 512 TMEM columns (two 128 x 256 fp32 accumulators) and issues the MMAs;
//   warps 2-5   write the one-hot A block [128 frames x 64] in the 128B-swizzled K-major layout
//               straight from the codes (one frame row per thread);
//   warps 6-9   epilogue: TMEM -> registers -> output (streaming stores); with RMSNorm they store
//               x and the frame's sum of squares over the 256 columns, and a second kernel
//               scales each row once all 24 partial sums are known.
// CUDA-core path (any other request): one block per frame, 80-row gather-sum in fp32.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dmel {
namespace {

// ---------------------------------------------------------------- element helpers

__device__ __forceinline__ void load8(const float *p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
  const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ void store8(float *p, const float (&v)[8]) {
  __stcs(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
  __stcs(reinterpret_cast<float4 *>(p) + 1, make_float4(v[4], v[5], v[6], v[7]));
}

__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&v)[8]) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]);
  u.w = pack_bf16x2(v[6], v[7]);
  __stcs(reinterpret_cast<uint4 *>(p), u);
}

// 16 bytes of output values: 4 fp32 (x[0..3]) or 8 bf16 (x[0..7], round to nearest even).
template <typename OT>
__device__ __forceinline__ uint4 pack16(const float (&x)[8]);
template <>
__device__ __forceinline__ uint4 pack16<float>(const float (&x)[8]) {
  return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
}
template <>
__device__ __forceinline__ uint4 pack16<__nv_bfloat16>(const float (&x)[8]) {
  return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                    pack_bf16x2(x[6], x[7]));
}

// Streaming (evict-first) 16-byte store.
template <typename OT>
__device__ __forceinline__ void st_stream16(OT *p, uint4 w) {
  __stcs(reinterpret_cast<uint4 *>(p), w);
}

__device__ __forceinline__ void load8_out(const float *p, float (&v)[8]) {
  const float4 a = __ldcs(reinterpret_cast<const float4 *>(p));
  const float4 b = __ldcs(reinterpret_cast<const float4 *>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load8_out(const __nv_bfloat16 *p, float (&v)[8]) {
  const uint4 u = __ldcs(reinterpret_cast<const uint4 *>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// ---------------------------------------------------------------- output rows

// Where frame f's vector goes: row f of out, or row rows[f] of an out with n_rows rows (the
// decoder's input sequence, frames spliced at their sentinels' expanded positions). A row
// outside [0, n_rows) is not written and is recorded as DMEL_DEVERR_OUT_ROW.
struct OutMap {
  const int64_t *rows;
  int64_t n_rows;
};

__device__ __forceinline__ int64_t map_row(const OutMap &om, int64_t f, uint32_t *err) {
  if (!om.rows) return f;
  const int64_t r = __ldg(om.rows + f);
  if (r < 0 || r >= om.n_rows) {
    if (err) record_error(err, DMEL_DEVERR_OUT_ROW);
    return -1;
  }
  return r;
}

// ---------------------------------------------------------------- CUDA-core path

constexpr int kSimtThreads = 256;
constexpr int kSimtMaxDim = 16384;

template <typename TT, typename OT>
__global__ void __launch_bounds__(kSimtThreads) embed_simt_kernel(const uint8_t *__restrict__ codes, int64_t F,
                                                                  const TT *__restrict__ table, int D,
                                                                  const TT *__restrict__ g, float eps,
                                                                  OT *__restrict__ out, OutMap om, uint32_t *err) {
  extern __shared__ __align__(16) float xs[];  // [D] when RMSNorm is on
  __shared__ int rows[kMel];
  __shared__ float red[kSimtThreads / 32];
  const int nv = D / 8;
  for (int64_t f = blockIdx.x; f < F; f += gridDim.x) {
    if (threadIdx.x < kMel) {
      int c = codes[f * kMel + threadIdx.x];
      if (c > 15) {
        record_error(err, DMEL_DEVERR_CODE_RANGE);
        c &= 15;
      }
      rows[threadIdx.x] = kLev * threadIdx.x + c;
    }
    const int64_t orow = map_row(om, f, threadIdx.x == 0 ? err : nullptr);
    __syncthreads();
    float ss = 0.0f;
    for (int v = threadIdx.x; v < nv; v += kSimtThreads) {
      float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int b = 0; b < kMel; ++b) {
        float t[8];
        load8(table + (size_t)rows[b] * D + 8 * v, t);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += t[i];
      }
      if (g) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          xs[8 * v + i] = acc[i];
          ss += acc[i] * acc[i];
        }
      } else if (orow >= 0) {
        store8(out + orow * D + 8 * v, acc);
      }
    }
    if (g) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
      __syncthreads();
      float tot = 0.0f;
#pragma unroll
      for (int w = 0; w < kSimtThreads / 32; ++w) tot += red[w];
      const float inv = 1.0f / sqrtf(tot / (float)D + eps);
      for (int v = threadIdx.x; v < nv; v += kSimtThreads) {
        float gv[8], y[8];
        load8(g + 8 * v, gv);
#pragma unroll
        for (int i = 0; i < 8; ++i) y[i] = gv[i] * (xs[8 * v + i] * inv);
        if (orow >= 0) store8(out + orow * D + 8 * v, y);
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- RMSNorm row scaling

// One warp per frame: ss = sum of the n_ct partial sums of squares, then
// out_j <- g_j * (out_j / sqrt(ss / D + eps)) in place.
constexpr int tc_bm = 128;  // frames per tile of the tensor-core kernel (partials layout)
template <typename OT>
__global__ void __launch_bounds__(256) rms_rescale_kernel(OT *__restrict__ out, OutMap om, int64_t F, int D,
                                                          const __nv_bfloat16 *__restrict__ g,
                                                          const float *__restrict__ partials, int n_ct, float eps) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t f = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); f < F; f += warps) {
    float ss = 0.0f;
    const float *col = partials + (f / tc_bm) * n_ct * tc_bm + (f % tc_bm);  // [frame tile][column tile][row]
    for (int c = lane; c < n_ct; c += 32) ss += col[(int64_t)c * tc_bm];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.0f / sqrtf(ss / (float)D + eps);
    const int64_t orow = map_row(om, f, nullptr);  // the embedding kernel recorded bad rows
    if (orow < 0) continue;
    OT *row = out + orow * D;
    for (int v = lane; v < D / 8; v += 32) {
      float x[8], gv[8], y[8];
      load8_out(row + 8 * v, x);
      load8(g + 8 * v, gv);
#pragma unroll
      for (int i = 0; i < 8; ++i) y[i] = gv[i] * (x[i] * inv);
      store8(row + 8 * v, y);
    }
  }
}

// ---------------------------------------------------------------- tensor-core path

namespace tc {
constexpr int BM = 128;                       // frames per tile (TMEM lanes)
constexpr int BN = 256;                       // table columns per tile
constexpr int BK = 64;                        // K per pipeline stage: 4 channels x 16 levels
constexpr int STAGES = 4;
constexpr int KBLOCKS = kRows / BK;           // 20
constexpr int A_STAGE = BM * BK * 2;          // 16 KB one-hot block
constexpr int B_BOX = BK * 64 * 2;            // 8 KB: 64 K-rows x 64 columns
constexpr int B_STAGE = BK * BN * 2;          // 32 KB table block
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
constexpr int OFF_BAR = OFF_B + STAGES * B_STAGE;
constexpr int N_BARS = 4 * STAGES + 5;
constexpr int OFF_G = OFF_BAR + 256;          // 256 fp32 RMSNorm weights of the block's columns
constexpr int SMEM_USED = OFF_G + BN * 4;
constexpr int SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack for the 1024-B swizzle atoms
constexpr int THREADS = 320;
constexpr uint32_t TMEM_COLS = 2 * BN;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
}  // namespace tc

// Epilogue variants of the tensor-core kernel.
enum TcMode : int {
  kPlain = 0,     // no RMSNorm: store x
  kPartials = 1,  // store x and each row's sum of squares over the tile (rms_rescale_kernel follows)
  kFused = 2,     // groups of D/256 blocks exchange the row sums and store the normalised rows
  kScaled = 3     // every row's RMSNorm scale is given (computed from the codes beforehand)
};

__device__ __forceinline__ void epi_barrier() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Barrier of the 128 epilogue threads that also ANDs a flag across them, so every epilogue
// thread takes the same branch after a bounded wait.
__device__ __forceinline__ bool epi_barrier_and(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(out)
      : "r"((uint32_t)v)
      : "memory");
  return out != 0;
}

__device__ __forceinline__ int ld_acquire(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Tile i of this block's schedule: (frame tile m, column tile nt). kPlain / kPartials walk all
// tiles with stride gridDim.x; kFused gives each block a fixed column tile (blockIdx % P) and
// makes each group of P consecutive blocks walk the same frame tiles.
template <int kMode>
__device__ __forceinline__ bool tile_at(int64_t i, int64_t n_m_tiles, int P, int64_t &m, int &nt) {
  if (kMode == kFused) {
    const int64_t G = gridDim.x / P;
    m = blockIdx.x / P + i * G;
    nt = blockIdx.x % P;
    return m < n_m_tiles;
  }
  const int64_t t = blockIdx.x + i * (int64_t)gridDim.x;
  m = t / P;
  nt = (int)(t % P);
  return m < n_m_tiles;
}

template <typename OT, int kMode>
__global__ void __launch_bounds__(tc::THREADS, 1)
    embed_tc_kernel(const __grid_constant__ CUtensorMap tmap, const uint8_t *__restrict__ codes, int64_t F, int D,
                    OT *__restrict__ out, OutMap om, float *__restrict__ partials, int *__restrict__ counters,
                    const __nv_bfloat16 *__restrict__ gw, float eps, uint32_t *err) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base, as an offset from the shared array (keeps the shared address space)
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  const uint32_t bar0 = smem_addr(bars);
  auto full_a = [&](int s) { return bar0 + 8u * s; };
  auto full_b = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto empty = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
  auto tfull = [&](int a) { return bar0 + 8u * (3 * STAGES + a); };
  auto tempty = [&](int a) { return bar0 + 8u * (3 * STAGES + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (3 * STAGES + 4);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_BAR + N_BARS * 8);
  float *gsm = reinterpret_cast<float *>(smem + OFF_G);  // RMSNorm weight of this block's columns

  const int P = D / BN;  // column tiles per row
  const int64_t n_m_tiles = (F + BM - 1) / BM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_a(s), 128);
      mbar_init(full_b(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), 128);
    }
    mbar_init(done_bar, 1);
    mbar_fence_init();
  }
  if (kMode == kFused && threadIdx.x < BN) {
    const int nt = blockIdx.x % P;
    gsm[threadIdx.x] = __bfloat162float(gw[nt * BN + threadIdx.x]);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmap);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer: table blocks
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t pending = 0;        // stages with a load issued
      uint32_t pending_phase = 0;  // phase bit of that load, per stage
      bool ok = true;
      int64_t m;
      int nt;
      for (int64_t i = 0; ok && tile_at<kMode>(i, n_m_tiles, P, m, nt); ++i) {
        const int n0 = nt * BN;
        for (int kb = 0; kb < KBLOCKS; ++kb) {
          if (!mbar_wait(empty(stage), phase ^ 1u, err)) { ok = false; break; }
          mbar_arrive_expect_tx(full_b(stage), B_STAGE);
          const uint32_t dst = smem_addr(smem + OFF_B + stage * B_STAGE);
#pragma unroll
          for (int q = 0; q < BN / 64; ++q) tma_load_2d(dst + q * B_BOX, &tmap, n0 + 64 * q, kb * BK, full_b(stage), pol);
          pending |= 1u << stage;
          pending_phase = (pending_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // every load issued must land before the block may exit
      for (int s = 0; s < STAGES; ++s)
        if (pending & (1u << s)) mbar_wait(full_b(s), (pending_phase >> s) & 1u, err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, 1);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int64_t m;
      int nt;
      for (int64_t i = 0; ok && tile_at<kMode>(i, n_m_tiles, P, m, nt); ++i) {
        const uint32_t acc = i & 1, acc_phase = (i >> 1) & 1;
        if (!mbar_wait(tempty(acc), acc_phase ^ 1u, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < KBLOCKS; ++kb) {
          if (!mbar_wait(full_a(stage), phase, err) || !mbar_wait(full_b(stage), phase, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_addr(smem + OFF_A + stage * A_STAGE);
          const uint32_t b0 = smem_addr(smem + OFF_B + stage * B_STAGE);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // A: K-major, 128B swizzle, 8-row groups 1024 B apart; K advances 32 B per step.
            const uint64_t adesc = smem_desc(a0 + 32u * k, 16u, 1024u, kSwizzle128B);
            // B: MN-major, 128B swizzle; 64-column boxes 8 KB apart (LBO), 8-row K groups
            // 1024 B apart (SBO); K advances 16 rows = 2 KB per step.
            const uint64_t bdesc = smem_desc(b0 + 2048u * k, (uint32_t)B_BOX, 1024u, kSwizzle128B);
            tc_mma_f16(d_tmem, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit(empty(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull(acc));
      }
      tc_commit(done_bar);
      mbar_wait(done_bar, 0, err);
    }
  } else if (warp < 6) {
    // ------------------------------------------------ one-hot A producers (row r per thread)
    const int r = threadIdx.x - 64;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int64_t m;
    int nt;
    for (int64_t i = 0; ok && tile_at<kMode>(i, n_m_tiles, P, m, nt); ++i) {
      const int64_t f = m * BM + r;
      uint32_t cw[20];
      const bool valid = f < F;
      if (valid) {
        const uint4 *src = reinterpret_cast<const uint4 *>(codes + f * kMel);
#pragma unroll
        for (int q = 0; q < 5; ++q) {
          const uint4 u = __ldg(src + q);
          cw[4 * q] = u.x; cw[4 * q + 1] = u.y; cw[4 * q + 2] = u.z; cw[4 * q + 3] = u.w;
        }
        uint32_t bad = 0;
#pragma unroll
        for (int q = 0; q < 20; ++q) bad |= cw[q] & 0xF0F0F0F0u;
        if (bad) record_error(err, DMEL_DEVERR_CODE_RANGE);
      } else {
#pragma unroll
        for (int q = 0; q < 20; ++q) cw[q] = 0;
      }
      const uint32_t row_off = (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u;
#pragma unroll
      for (int kb = 0; kb < KBLOCKS; ++kb) {
        if (!mbar_wait(empty(stage), phase ^ 1u, err)) { ok = false; break; }
        uint8_t *rowp = smem + OFF_A + stage * A_STAGE + row_off;
        const uint32_t w = cw[kb];  // codes of channels 4 kb .. 4 kb + 3
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          // 16-byte chunk ch holds levels 8 (ch & 1) .. +7 of channel 4 kb + (ch >> 1)
          const uint32_t c = (w >> (8 * (ch >> 1))) & 15u;
          const bool hit = valid && ((c >> 3) == (uint32_t)(ch & 1));
          const uint32_t e = c & 7u;
          const uint32_t one = (e & 1u) ? 0x3F800000u : 0x00003F80u;  // bf16 1.0 in the low or high half
          uint4 v;
          v.x = (hit && (e >> 1) == 0) ? one : 0u;
          v.y = (hit && (e >> 1) == 1) ? one : 0u;
          v.z = (hit && (e >> 1) == 2) ? one : 0u;
          v.w = (hit && (e >> 1) == 3) ? one : 0u;
          *reinterpret_cast<uint4 *>(rowp + ((ch ^ (r & 7)) << 4)) = v;  // 128B swizzle
        }
        fence_proxy_async_smem();
        mbar_arrive(full_a(stage));
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else {
    // ------------------------------------------------ epilogue (TMEM lanes 32 (warp % 4) ..)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    bool ok = true;
    int64_t m;
    int nt;
    for (int64_t i = 0; ok && tile_at<kMode>(i, n_m_tiles, P, m, nt); ++i) {
      const uint32_t acc = i & 1, acc_phase = (i >> 1) & 1;
      if (!epi_barrier_and(mbar_wait(tfull(acc), acc_phase, err))) { ok = false; break; }
      tc_fence_after();
      const int64_t f = m * BM + r;
      const bool valid = f < F;
      const int64_t row = valid ? map_row(om, f, err) : -1;
      OT *orow = out + (row >= 0 ? row : 0) * (int64_t)D + nt * BN;
      const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * BN;
      float scale = 1.0f;
      if (kMode != kPlain) {
        // the row's sum of squares over this tile's 256 columns
        float ss = 0.0f;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v0[16], v1[16];
          tmem_ld16(tbase + c * 32, v0);
          tmem_ld16(tbase + c * 32 + 16, v1);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float a = __uint_as_float(v0[q]), b = __uint_as_float(v1[q]);
            ss = fmaf(a, a, ss);
            ss = fmaf(b, b, ss);
          }
        }
        float *slot = partials + ((m * P + nt) * BM);
        if (kMode == kPartials) {
          slot[r] = ss;
        } else {
          // publish this tile's row sums, wait until the group's P column tiles have all
          // published theirs (bounded), then add them in a fixed order
          __stcg(slot + r, ss);
          __threadfence();
          epi_barrier();
          if (r == 0) {
            atomicAdd(counters + m, 1);
            uint32_t polls = 0;
            while (ld_acquire(counters + m) < P) {
              if (++polls > kMaxPolls) {
                record_error(err, DMEL_DEVERR_WAIT_TIMEOUT);
                break;
              }
              __nanosleep(32);
            }
          }
          epi_barrier();
          __threadfence();
          const float *col = partials + m * P * BM + r;
          float tot = 0.0f;
          for (int q = 0; q < P; ++q) tot += __ldcg(col + q * BM);
          scale = 1.0f / sqrtf(tot / (float)D + eps);
        }
      }
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v0[16], v1[16];
        tmem_ld16(tbase + c * 32, v0);
        tmem_ld16(tbase + c * 32 + 16, v1);
        tmem_wait_ld();
        if (row >= 0) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            float x[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const uint32_t u = h < 2 ? v0[8 * h + q] : v1[8 * (h - 2) + q];
              x[q] = __uint_as_float(u);
              if (kMode == kFused) x[q] = gsm[c * 32 + 8 * h + q] * (x[q] * scale);
            }
            store8(orow + c * 32 + 8 * h, x);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty(acc));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- tensor-core path, CTA pairs

// A cluster of two CTAs computes a 256-frame x 256-column tile with tcgen05.mma.cta_group::2:
// each CTA writes the one-hot rows of its own 128 frames and loads half of the table block
// (128 columns), the even CTA issues the MMAs for both, and each CTA's TMEM receives its 128
// rows x 256 columns. Per SM this halves the table traffic from L2 and the operand bytes the
// tensor core reads from shared memory, compared with the one-CTA tile.
namespace tc2 {
constexpr int BM = 128;                      // frames per CTA
constexpr int BN = 256;                      // columns per pair tile
constexpr int BNH = 128;                     // columns loaded by each CTA
constexpr int BK = 64;
constexpr int STAGES = 6;
constexpr int KBLOCKS = kRows / BK;
constexpr int A_STAGE = BM * BK * 2;         // 16 KB
constexpr int B_BOX = BK * 64 * 2;           // 8 KB
constexpr int B_STAGE = BK * BNH * 2;        // 16 KB
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
constexpr int OFF_BAR = OFF_B + STAGES * B_STAGE;
constexpr int N_BARS = 3 * STAGES + 5;
constexpr int OFF_G = OFF_BAR + 256;
constexpr int SMEM_USED = OFF_G + BN * 4;
constexpr int SMEM_BYTES = SMEM_USED + 1024;
constexpr int THREADS = 320;
constexpr uint32_t TMEM_COLS = 2 * BN;
static_assert(N_BARS * 8 + 16 <= 256, "barrier area");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
}  // namespace tc2

// Pair tile i of this cluster: (pair frame tile mp, column tile nt). kPlain / kPartials walk all
// pair tiles with stride = number of clusters; kFused gives each cluster a fixed column tile
// and makes each group of P clusters walk the same pair frame tiles.
template <int kMode>
__device__ __forceinline__ bool pair_tile_at(int64_t i, int64_t n_pm, int P, int64_t &mp, int &nt) {
  const int64_t cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  if (kMode == kFused) {
    const int64_t G = ncl / P;
    mp = cid / P + i * G;
    nt = (int)(cid % P);
    return mp < n_pm;
  }
  const int64_t t = cid + i * ncl;
  mp = t / P;
  nt = (int)(t % P);
  return mp < n_pm;
}

template <typename OT, int kMode>
__global__ void __launch_bounds__(tc2::THREADS, 1)
    embed_tc2_kernel(const __grid_constant__ CUtensorMap tmap, const uint8_t *__restrict__ codes, int64_t F, int D,
                     OT *__restrict__ out, OutMap om, float *__restrict__ partials, int *__restrict__ counters,
                     const __nv_bfloat16 *__restrict__ gw, float eps, uint32_t *err) {
  using namespace tc2;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base, as an offset from the shared array (keeps the shared address space)
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  const uint32_t bar0 = smem_addr(bars);
  auto full_a = [&](int s) { return bar0 + 8u * s; };
  auto full_b = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto empty = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
  auto tfull = [&](int a) { return bar0 + 8u * (3 * STAGES + a); };
  auto tempty = [&](int a) { return bar0 + 8u * (3 * STAGES + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (3 * STAGES + 4);
  auto in_leader = [&](uint32_t local_bar) { return mapa_shared(local_bar, 0); };
  auto in_peer = [&](uint32_t local_bar) { return mapa_shared(local_bar, 1); };
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_BAR + N_BARS * 8);
  float *gsm = reinterpret_cast<float *>(smem + OFF_G);

  const int P = D / BN;
  const int64_t n_m_tiles = (F + BM - 1) / BM;      // 128-frame tiles with at least one frame
  const int64_t n_pm = (F + 2 * BM - 1) / (2 * BM);  // 256-frame pair tiles

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_a(s), 8);  // 4 producer warps of each CTA (used in the even CTA)
      mbar_init(full_b(s), 1);  // the leader's expect-tx for both halves
      mbar_init(empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), 8);  // 4 epilogue warps of each CTA (used in the even CTA)
    }
    mbar_init(done_bar, 1);
    mbar_fence_init();
  }
  if (kMode == kFused && threadIdx.x < BN) {
    const int nt = (int)((blockIdx.x >> 1) % P);
    gsm[threadIdx.x] = __bfloat162float(gw[nt * BN + threadIdx.x]);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_addr(tmem_holder), TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmap);
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer: this CTA's half of the table block
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t pending = 0, pending_phase = 0;
      bool ok = true;
      int64_t mp;
      int nt;
      for (int64_t i = 0; ok && pair_tile_at<kMode>(i, n_pm, P, mp, nt); ++i) {
        const int n0 = nt * BN + (int)rank * BNH;
        for (int kb = 0; kb < KBLOCKS; ++kb) {
          if (!mbar_wait(empty(stage), phase ^ 1u, err)) { ok = false; break; }
          const uint32_t fb = in_leader(full_b(stage));
          if (leader) mbar_arrive_expect_tx(full_b(stage), 2 * B_STAGE);  // both CTAs' halves
          const uint32_t dst = smem_addr(smem + OFF_B + stage * B_STAGE);
#pragma unroll
          for (int q = 0; q < BNH / 64; ++q) tma_load_2d_pair(dst + q * B_BOX, &tmap, n0 + 64 * q, kb * BK, fb, pol);
          pending |= 1u << stage;
          pending_phase = (pending_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // the leader's MMA thread consumes every load; the leader waits for the last ones below
      if (leader)
        for (int s = 0; s < STAGES; ++s)
          if (pending & (1u << s)) mbar_wait(full_b(s), (pending_phase >> s) & 1u, err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (even CTA only)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN, 1);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int64_t mp;
      int nt;
      for (int64_t i = 0; ok && pair_tile_at<kMode>(i, n_pm, P, mp, nt); ++i) {
        const uint32_t acc = i & 1, acc_phase = (i >> 1) & 1;
        if (!mbar_wait(tempty(acc), acc_phase ^ 1u, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < KBLOCKS; ++kb) {
          if (!mbar_wait(full_a(stage), phase, err) || !mbar_wait(full_b(stage), phase, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_addr(smem + OFF_A + stage * A_STAGE);
          const uint32_t b0 = smem_addr(smem + OFF_B + stage * B_STAGE);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t adesc = smem_desc(a0 + 32u * k, 16u, 1024u, kSwizzle128B);
            const uint64_t bdesc = smem_desc(b0 + 2048u * k, (uint32_t)B_BOX, 1024u, kSwizzle128B);
            tc_mma_f16_pair(d_tmem, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit_pair(empty(stage));
          tc_commit_pair(in_peer(empty(stage)));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair(tfull(acc));
        tc_commit_pair(in_peer(tfull(acc)));
      }
      tc_commit_pair(done_bar);
      mbar_wait(done_bar, 0, err);
    }
  } else if (warp < 6) {
    // ------------------------------------------------ one-hot A producers (row r per thread)
    const int r = threadIdx.x - 64;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int64_t mp;
    int nt;
    for (int64_t i = 0; ok && pair_tile_at<kMode>(i, n_pm, P, mp, nt); ++i) {
      const int64_t f = (2 * mp + rank) * BM + r;
      uint32_t cw[20];
      const bool valid = f < F;
      if (valid) {
        const uint4 *src = reinterpret_cast<const uint4 *>(codes + f * kMel);
#pragma unroll
        for (int q = 0; q < 5; ++q) {
          const uint4 u = __ldg(src + q);
          cw[4 * q] = u.x; cw[4 * q + 1] = u.y; cw[4 * q + 2] = u.z; cw[4 * q + 3] = u.w;
        }
        uint32_t bad = 0;
#pragma unroll
        for (int q = 0; q < 20; ++q) bad |= cw[q] & 0xF0F0F0F0u;
        if (bad) record_error(err, DMEL_DEVERR_CODE_RANGE);
      } else {
#pragma unroll
        for (int q = 0; q < 20; ++q) cw[q] = 0;
      }
      const uint32_t row_off = (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u;
#pragma unroll
      for (int kb = 0; kb < KBLOCKS; ++kb) {
        if (!mbar_wait(empty(stage), phase ^ 1u, err)) { ok = false; break; }
        uint8_t *rowp = smem + OFF_A + stage * A_STAGE + row_off;
        const uint32_t w = cw[kb];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint32_t c = (w >> (8 * (ch >> 1))) & 15u;
          const bool hit = valid && ((c >> 3) == (uint32_t)(ch & 1));
          const uint32_t e = c & 7u;
          const uint32_t one = (e & 1u) ? 0x3F800000u : 0x00003F80u;
          uint4 v;
          v.x = (hit && (e >> 1) == 0) ? one : 0u;
          v.y = (hit && (e >> 1) == 1) ? one : 0u;
          v.z = (hit && (e >> 1) == 2) ? one : 0u;
          v.w = (hit && (e >> 1) == 3) ? one : 0u;
          *reinterpret_cast<uint4 *>(rowp + ((ch ^ (r & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(in_leader(full_a(stage)));
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else {
    // ------------------------------------------------ epilogue (this CTA's 128 rows)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    bool ok = true;
    int64_t mp;
    int nt;
    for (int64_t i = 0; ok && pair_tile_at<kMode>(i, n_pm, P, mp, nt); ++i) {
      const uint32_t acc = i & 1, acc_phase = (i >> 1) & 1;
      if (!epi_barrier_and(mbar_wait(tfull(acc), acc_phase, err))) { ok = false; break; }
      tc_fence_after();
      const int64_t m = 2 * mp + rank;
      const int64_t f = m * BM + r;
      const bool valid = f < F;
      const bool live = m < n_m_tiles;  // the pair's second half may hold no frame at all
      const int64_t row = valid ? map_row(om, f, err) : -1;
      OT *orow = out + (row >= 0 ? row : 0) * (int64_t)D + nt * BN;
      const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * BN;
      float scale = 1.0f;
      if (kMode != kPlain && live) {
        float ss = 0.0f;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v0[16], v1[16];
          tmem_ld16(tbase + c * 32, v0);
          tmem_ld16(tbase + c * 32 + 16, v1);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float a = __uint_as_float(v0[q]), b = __uint_as_float(v1[q]);
            ss = fmaf(a, a, ss);
            ss = fmaf(b, b, ss);
          }
        }
        float *slot = partials + ((m * P + nt) * BM);
        if (kMode == kPartials) {
          slot[r] = ss;
        } else {
          __stcg(slot + r, ss);
          __threadfence();
          epi_barrier();
          if (r == 0) {
            atomicAdd(counters + m, 1);
            uint32_t polls = 0;
            while (ld_acquire(counters + m) < P) {
              if (++polls > kMaxPolls) {
                record_error(err, DMEL_DEVERR_WAIT_TIMEOUT);
                break;
              }
              __nanosleep(32);
            }
          }
          epi_barrier();
          __threadfence();
          const float *col = partials + m * P * BM + r;
          float tot = 0.0f;
          for (int q = 0; q < P; ++q) tot += __ldcg(col + q * BM);
          scale = 1.0f / sqrtf(tot / (float)D + eps);
        }
      }
      if (live) {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v0[16], v1[16];
          tmem_ld16(tbase + c * 32, v0);
          tmem_ld16(tbase + c * 32 + 16, v1);
          tmem_wait_ld();
          if (row >= 0) {
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              float x[8];
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const uint32_t u = h < 2 ? v0[8 * h + q] : v1[8 * (h - 2) + q];
                x[q] = __uint_as_float(u);
                if (kMode == kFused) x[q] = gsm[c * 32 + 8 * h + q] * (x[q] * scale);
              }
              store8(orow + c * 32 + 8 * h, x);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(in_leader(tempty(acc)));
    }
  }

  tc_fence_before();
  cluster_sync();  // every MMA into either CTA's TMEM has completed (the leader waited above)
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- 2:4-sparse one-hot product

// Each bin's 16 one-hot columns hold a single 1, so every group of four consecutive table rows
// has at most one non-zero in A: A is 2:4 sparse and tcgen05.mma.sp halves the tensor work.
// Per bin and frame with level c: A keeps two values out of each group of four rows (group
// c >> 2 keeps rows (0, 1) or (2, 3) of the group, whichever holds c; the other groups keep
// (0, 1) with zeros), so the 16 logical columns become 8 stored bf16 (16 bytes) with the 1 at
// position 2 (c >> 2) + (c & 1), and 16 bits of metadata (a nibble of two 2-bit row positions
// per group). The metadata lives in TMEM, one 32-bit column per MMA (logical K = 32, two bins).
// Tiles are 256 frames x 192 columns: two fp32 accumulators at TMEM columns 0 and 256, three
// 32-column A slots at 192, 224 and 448 and a three-stage metadata ring at 480..491. With
// RMSNorm, groups of ceil(D / 192) clusters (32 at D = 6144, two groups, 64 clusters, on 148
// SMs) own fixed column slices and walk the same frame tiles together; each row's sum of squares
// over a slice is published into a buffer pre-filled with a sentinel and the other slices'
// sums are read as they appear (all clusters are co-resident under the cooperative launch).
// An mbarrier wait in the thread that issues tcgen05.mma stalls that thread behind its queued
// MMAs and leaves the tensor pipe idle for a few hundred cycles per wait, so a separate warp does
// every wait and hands each stage to the MMA warp through named barriers, running up to three
// stages ahead (a wait that times out is recorded and the waiter stops waiting but keeps
// handing over stages, so the kernel finishes).
// Each commit signals the barrier in both CTAs at once. Eight epilogue warps (two
// per TMEM lane quarter, 96 columns each) stage their rows in shared memory and write whole
// 64-byte (bf16) or 128-byte (fp32) row pieces, 8 or 4 rows per warp instruction.
namespace sp {
constexpr int BM = 128;                 // frames per CTA
constexpr int BN = 192;                 // columns per pair tile
constexpr int BNH = 96;                 // columns used from each CTA's half of the table block
constexpr int BKL = 128;                // table rows (logical K) per stage: 8 bins
constexpr int KBLOCKS = kRows / BKL;    // 10
constexpr int STAGES_A = 3;             // A + metadata slots in TMEM
constexpr int STAGES_B = 7;             // table blocks in shared memory
constexpr int B_BOX_COLS = 32;          // 64-byte rows, 64-byte swizzle
constexpr int B_BOXES = BNH / B_BOX_COLS;
constexpr int B_BOX = B_BOX_COLS * BKL * 2;  // 32 columns x 128 rows: 8 KB
constexpr int B_STAGE = B_BOXES * B_BOX;     // exactly the 96 columns used
constexpr int OFF_B = 0;
constexpr int OFF_BAR = OFF_B + STAGES_B * B_STAGE;
constexpr int N_BARS = 2 * STAGES_A + 2 * STAGES_B + 5;
constexpr int BN_EPI = BN;              // columns the epilogue walks
constexpr int EPI_WARPS = 8;            // two per TMEM lane quarter
constexpr int EPI_COLS = BN / 2;        // columns per epilogue warp
constexpr int EPI_CHUNK = 32;           // columns staged at a time
constexpr int OFF_G = OFF_BAR + 256;    // RMSNorm weights of the column tile (kScaled: [2], by accumulator)
constexpr int OFF_EPI = OFF_G + 2 * BN_EPI * 4;  // row sums [2][128] and scales [128]
constexpr int OFF_STG = OFF_EPI + 3 * BM * 4;  // staging: 8 warps x 32 rows x up to 128 bytes
constexpr int OFF_RING = OFF_STG + EPI_WARPS * 32 * 128;  // dynamic schedule: {tile index, sequence} [16]
constexpr int RING = 16;
constexpr int LOOKAHEAD = 3;  // tiles published ahead of the one the TMA warp starts
constexpr int OFF_ATAB = OFF_RING + RING * 8;  // one bin's 4 stored A words by level, + a zero row
constexpr int OFF_MTAB = OFF_ATAB + 17 * 16;   // metadata of two bins by their levels [256]
constexpr int SMEM_USED = OFF_MTAB + 256 * 4;
constexpr int SMEM_BYTES = SMEM_USED + 1024;
constexpr int WAITER_WARP = 6 + EPI_WARPS;  // warps: 0 TMA, 1 MMA, 2..5 A, 6..13 epilogue, 14 waits
constexpr int THREADS = 32 * (WAITER_WARP + 1);
// TMEM columns: accumulators [0, 192) and [256, 448); A slots (32 columns: 64 stored bf16 per
// row) at 192, 224, 448; metadata slots (4 columns) at 480, 484, 488.
constexpr uint32_t ACC_STRIDE = 256;
__host__ __device__ constexpr uint32_t a_col(int s) { return s == 0 ? 192u : s == 1 ? 224u : 448u; }
constexpr uint32_t META_COL = 480;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t kSentinel = 0xFFFFFFFFu;  // a NaN no arithmetic produces: "not yet published"
constexpr uint32_t kBackoffNs = 256;          // sleep between polls of the waits with slack
static_assert(KBLOCKS * BKL == kRows, "stages cover the table");
static_assert(BN % 64 == 0 && BN <= 192, "accumulator columns end where the A slots start");
static_assert(STAGES_A == 3 && META_COL >= 448 + 32 && META_COL + 4 * STAGES_A <= TMEM_COLS, "TMEM map");
static_assert(N_BARS * 8 + 16 <= 256, "barrier area");
static_assert(B_BOXES * B_BOX_COLS == BNH && B_STAGE % 1024 == 0 && STAGES_B <= 32, "table stages");
static_assert(OFF_STG % 128 == 0, "staging rows are 128-byte aligned");
static_assert(EPI_COLS % EPI_CHUNK == 0 && EPI_CHUNK == 32, "epilogue slices");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
}  // namespace sp

// Named barrier 1 over the sparse kernel's 8 epilogue warps; the _and form returns whether v held
// in every thread. Named barrier 2 joins the waiter warp and the MMA warp once per stage.
__device__ __forceinline__ void sp_epi_barrier() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ bool sp_epi_barrier_and(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(out)
      : "r"((uint32_t)v)
      : "memory");
  return out != 0;
}
// Stage handoff between the waiter warp and the MMA warp: named barriers 2..4 ("stage j is
// ready", waiter arrives, MMA warp syncs) and 5..7 ("stage j was issued", MMA warp arrives,
// waiter syncs), j = stage mod 3. The waiter announces stage s + 3 only after the MMA warp
// acknowledged stage s, so it runs at most three stages ahead and never arrives twice on a
// barrier the MMA warp has not yet consumed.
__device__ __forceinline__ void sp_ready_arrive(int j) { asm volatile("bar.arrive %0, 64;" ::"r"(2 + j) : "memory"); }
__device__ __forceinline__ void sp_ready_sync(int j) { asm volatile("bar.sync %0, 64;" ::"r"(2 + j) : "memory"); }
__device__ __forceinline__ void sp_issued_arrive(int j) { asm volatile("bar.arrive %0, 64;" ::"r"(5 + j) : "memory"); }
__device__ __forceinline__ void sp_issued_sync(int j) { asm volatile("bar.sync %0, 64;" ::"r"(5 + j) : "memory"); }

__device__ __forceinline__ void st_relaxed_f32(float *p, float v) {
  asm volatile("st.relaxed.gpu.global.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_relaxed_u32(const float *p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Number of column tiles of the sparse kernel (the last one may be partial).
__host__ __device__ constexpr int sp_col_tiles(int D) { return (D + sp::BN - 1) / sp::BN; }

// 8-byte shared-memory slots of either CTA of the cluster (addresses from mapa_shared) for the
// tile index ring of the dynamic schedule: one aligned 8-byte access is single-copy atomic, so a
// slot carries its own sequence number and needs no release/acquire pairing with a second word.
__device__ __forceinline__ void st_relaxed_cluster_u64(uint32_t cluster_addr, unsigned long long v) {
  asm volatile("st.relaxed.cluster.shared::cluster.u64 [%0], %1;" ::"r"(cluster_addr), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_cluster_u64(uint32_t local_addr) {
  unsigned long long v;
  asm volatile("ld.relaxed.cluster.shared::cta.u64 %0, [%1];" : "=l"(v) : "r"(local_addr) : "memory");
  return v;
}

// Tile i of this cluster: pair frame tile mp, column tile nt. Without RMSNorm the clusters walk
// one global order (frame tile major); with it, groups of P clusters own fixed column slices
// and walk the same frame tiles.
template <int kMode>
__device__ __forceinline__ bool sp_tile_at(int64_t i, int64_t n_pm, int P, int64_t &mp, int &nt) {
  const int64_t cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  if (kMode == kFused) {
    mp = cid / P + i * (ncl / P);
    nt = (int)(cid % P);
    return mp < n_pm;
  }
  const int64_t t = cid + i * ncl;
  mp = t / P;
  nt = (int)(t % P);
  return mp < n_pm;
}

// Metadata of one bin at level c: groups keep rows (0, 1) (nibble 0x4) except group c >> 2,
// which keeps (2, 3) (nibble 0xE) when c & 3 is 2 or 3.
__device__ __forceinline__ uint32_t sp_meta_field(uint32_t c) {
  return 0x4444u | ((c & 2u) ? (0xAu << (4u * (c >> 2))) : 0u);
}

template <typename OT, int kMode>
__global__ void __launch_bounds__(sp::THREADS, 1)
    embed_sp_kernel(const __grid_constant__ CUtensorMap tmap, const uint8_t *__restrict__ codes, int64_t F, int D,
                    OT *__restrict__ out, OutMap om, float *__restrict__ partials, int *__restrict__ counters,
                    const __nv_bfloat16 *__restrict__ gw, float eps, uint32_t *err) {
  using namespace sp;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base, as an offset from the shared array (keeps the shared address space)
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  const uint32_t bar0 = smem_addr(bars);
  auto full_a = [&](int s) { return bar0 + 8u * s; };
  auto empty_a = [&](int s) { return bar0 + 8u * (STAGES_A + s); };
  auto full_b = [&](int s) { return bar0 + 8u * (2 * STAGES_A + s); };
  auto empty_b = [&](int s) { return bar0 + 8u * (2 * STAGES_A + STAGES_B + s); };
  auto tfull = [&](int a) { return bar0 + 8u * (2 * STAGES_A + 2 * STAGES_B + a); };
  auto tempty = [&](int a) { return bar0 + 8u * (2 * STAGES_A + 2 * STAGES_B + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (2 * STAGES_A + 2 * STAGES_B + 4);
  auto in_leader = [&](uint32_t local_bar) { return mapa_shared(local_bar, 0); };
  auto in_peer = [&](uint32_t local_bar) { return mapa_shared(local_bar, 1); };
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_BAR + N_BARS * 8);
  float *gsm = reinterpret_cast<float *>(smem + OFF_G);

  const int P = sp_col_tiles(D);
  const int64_t n_m_tiles = (F + BM - 1) / BM;      // 128-frame tiles with at least one frame
  const int64_t n_pm = (F + 2 * BM - 1) / (2 * BM);  // 256-frame pair tiles

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES_A; ++s) {
      mbar_init(full_a(s), 8);  // 4 producer warps of each CTA (used in the even CTA)
      mbar_init(empty_a(s), 1);
    }
    for (int s = 0; s < STAGES_B; ++s) {
      mbar_init(full_b(s), 1);  // the leader's expect-tx for both halves
      mbar_init(empty_b(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), 2 * EPI_WARPS);  // epilogue warps of both CTAs (used in the even CTA)
    }
    mbar_init(done_bar, 1);
    if (kMode == kScaled)
      for (int q = 0; q < RING; ++q)  // dynamic schedule: nothing published (no sequence number matches)
        reinterpret_cast<unsigned long long *>(smem + OFF_RING)[q] = ~0ull;
    // a bin's 8 stored bf16 of A at level c: the 1 in column c >> 2 of the four 32-bit columns,
    // low half when c is even; row 16 is a frame past the end (no 1)
    uint32_t *atab = reinterpret_cast<uint32_t *>(smem + OFF_ATAB);
    for (int c = 0; c < 17; ++c)
      for (int g = 0; g < 4; ++g)
        atab[4 * c + g] = c < 16 && (c >> 2) == g ? ((c & 1) ? 0x3F800000u : 0x00003F80u) : 0u;
    mbar_fence_init();
  }
  // the metadata of two bins at levels c0 and c1, at index c0 + 16 c1
  for (int e = threadIdx.x; e < 256; e += blockDim.x)
    reinterpret_cast<uint32_t *>(smem + OFF_MTAB)[e] = sp_meta_field(e & 15) | (sp_meta_field(e >> 4) << 16);
  if (kMode == kFused && threadIdx.x < BN_EPI) {
    const int c = (int)((blockIdx.x >> 1) % P) * BN + threadIdx.x;
    gsm[threadIdx.x] = c < D ? __bfloat162float(gw[c]) : 0.0f;
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_addr(tmem_holder), TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmap);
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // Dynamic schedule (kScaled with a tile counter): the clusters take tiles from one global
  // counter, so clusters on faster SMs take more; the even CTA's TMA thread fetches the indices
  // and writes them, in order, into a ring in both CTAs' shared memory, and every role of both
  // CTAs reads tile i of the cluster from its own copy: slot i mod RING holds {tile index, i} in
  // one 8-byte word, so a reader polls that slot until it carries sequence number i (relaxed
  // loads: no acquire, which cost ~700 cycles per lookup at each tile boundary). The publisher
  // runs at most LOOKAHEAD tiles ahead of the TMA warp, which the stage barriers keep within a
  // few tiles of the slowest role, far inside the ring.
  const bool dyn = kMode == kScaled && counters != nullptr;
  const int64_t n_tiles_all = n_pm * (int64_t)P;
  const uint32_t ring_addr = smem_addr(smem + OFF_RING);
  auto tile = [&](int64_t i, int64_t &mp_, int &nt_) -> bool {
    if (!dyn) return sp_tile_at<kMode>(i, n_pm, P, mp_, nt_);
    const uint32_t slot = ring_addr + 8u * (uint32_t)(i & (RING - 1));
    uint32_t polls = 0;
    unsigned long long v;
    while ((uint32_t)((v = ld_relaxed_cluster_u64(slot)) >> 32) != (uint32_t)i) {
      if (++polls > kMaxPolls) {
        record_error(err, DMEL_DEVERR_WAIT_TIMEOUT);
        return false;
      }
    }
    const int t = (int)(uint32_t)v;
    if (t < 0 || (int64_t)t >= n_tiles_all) return false;
    mp_ = t / P;
    nt_ = t % P;
    return true;
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer: this CTA's half of the table block
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t pending = 0, pending_phase = 0;
      bool ok = true;
      int64_t mp;
      int nt;
      int64_t n_pub = 0;      // ring entries published (even CTA)
      bool pub_end = false;   // the entry past the last tile has been published
      auto publish_upto = [&](int64_t k) {
        while (dyn && leader && !pub_end && n_pub < k) {
          const int t = atomicAdd(counters, 1);
          const unsigned long long v = ((unsigned long long)(uint32_t)n_pub << 32) | (uint32_t)t;
          const uint32_t off = 8u * (uint32_t)(n_pub & (RING - 1));
          st_relaxed_cluster_u64(mapa_shared(ring_addr + off, 0), v);
          st_relaxed_cluster_u64(mapa_shared(ring_addr + off, 1), v);
          ++n_pub;
          pub_end = (int64_t)t >= n_tiles_all;
        }
      };
      publish_upto(1 + LOOKAHEAD);
      for (int64_t i = 0; ok && tile(i, mp, nt); ++i) {
        publish_upto(i + 1 + LOOKAHEAD);
        const int n0 = nt * BN + (int)rank * BNH;
        for (int kb = 0; kb < KBLOCKS; ++kb) {
          // the ring runs STAGES_B stages ahead of the MMAs: poll with sleeps, so this thread
          // leaves the issue slots to the A producers
          if (!mbar_wait_backoff(empty_b(stage), phase ^ 1u, err, kBackoffNs)) { ok = false; break; }
          const uint32_t fb = in_leader(full_b(stage));
          if (leader) mbar_arrive_expect_tx(full_b(stage), 2 * B_STAGE);  // both CTAs' halves
          const uint32_t dst = smem_addr(smem + OFF_B + stage * B_STAGE);
#pragma unroll
          for (int q = 0; q < B_BOXES; ++q)
            tma_load_2d_pair(dst + q * B_BOX, &tmap, n0 + B_BOX_COLS * q, kb * BKL, fb, pol);
          pending |= 1u << stage;
          pending_phase = (pending_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES_B) { stage = 0; phase ^= 1u; }
        }
      }
      if (leader)
        for (int s = 0; s < STAGES_B; ++s)
          if (pending & (1u << s)) mbar_wait(full_b(s), (pending_phase >> s) & 1u, err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA warp (even CTA only): lane 0 issues
    // Stage by stage the waiter warp reports (named barrier 2) that the accumulator, A slot and
    // table block are ready; this warp itself never waits on an mbarrier while MMAs are queued.
    if (leader) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN, 1) | kIdescSparse;
      int sa = 0, sb = 0;
      int64_t mp;
      int nt;
      for (int64_t i = 0; tile(i, mp, nt); ++i) {
        const uint32_t acc = i & 1;
        const uint32_t d_tmem = tmem_base + acc * ACC_STRIDE;
        for (int kb = 0; kb < KBLOCKS; ++kb) {
          sp_ready_sync(sa);  // A slot sa cycles with the stage index mod 3
          if (lane == 0) {
            tc_fence_after();
            const uint32_t b0 = smem_addr(smem + OFF_B + sb * B_STAGE);
            const uint32_t a0 = tmem_base + a_col(sa);
#pragma unroll
            for (int k = 0; k < BKL / 32; ++k) {
              // MN-major, 64-byte swizzle: atoms of 32 columns x 8 rows (512 bytes), boxes of 32
              // columns B_BOX apart; 32 table rows (2048 bytes) per MMA
              const uint64_t bdesc = smem_desc(b0 + 2048u * k, (uint32_t)B_BOX, 512u, kSwizzle64B);
              const uint32_t mcol = META_COL + 4u * sa + k;
              tc_mma_sp_pair_ts(d_tmem, a0 + 8u * k, bdesc, idesc | (mcol & 1u), tmem_base + (mcol & ~1u),
                                (kb | k) != 0 ? 1u : 0u);
            }
            tc_commit_pair_both(empty_a(sa), 3);
            tc_commit_pair_both(empty_b(sb), 3);
            if (kb == KBLOCKS - 1) tc_commit_pair_both(tfull(acc), 3);
          }
          __syncwarp();
          sp_issued_arrive(sa);
          if (++sa == STAGES_A) sa = 0;
          if (++sb == STAGES_B) sb = 0;
        }
      }
      if (lane == 0) {
        tc_commit_pair(done_bar);
        mbar_wait(done_bar, 0, err);
      }
    }
  } else if (warp == WAITER_WARP) {
    // ------------------------------------------------ waits for the MMA warp (even CTA only)
    if (leader) {
      int sa = 0, sb = 0;
      uint32_t pa = 0, pb = 0;
      bool ok = true;  // after a timed-out wait: no more waiting, stages still handed over
      int64_t n = 0;   // stages announced
      int64_t mp;
      int nt;
      for (int64_t i = 0; tile(i, mp, nt); ++i) {
        const uint32_t acc = i & 1, acc_phase = (i >> 1) & 1;
        for (int kb = 0; kb < KBLOCKS; ++kb, ++n) {
          if (n >= STAGES_A) sp_issued_sync(sa);  // stage n - 3 (same slot) was issued
          if (lane == 0 && ok) {
            // the table block is usually long resident: its wait first, the A slot's last
            if (kb == 0) ok = mbar_wait(tempty(acc), acc_phase ^ 1u, err);
            ok = ok && mbar_wait(full_b(sb), pb, err) && mbar_wait(full_a(sa), pa, err);
          }
          __syncwarp();
          sp_ready_arrive(sa);
          if (++sa == STAGES_A) { sa = 0; pa ^= 1u; }
          if (++sb == STAGES_B) { sb = 0; pb ^= 1u; }
        }
      }
      // consume the acknowledgements of the last stages (at most three), oldest first
      for (int64_t q = n > STAGES_A ? n - STAGES_A : 0; q < n; ++q) sp_issued_sync((int)(q % STAGES_A));
    }
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------ compressed one-hot A + metadata into TMEM
    // Warp w may only touch TMEM lanes 32 (w % 4) .. + 31, so it owns those rows (row r in lane r).
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    // Metadata lane order within the warp: lane t holds rows (t & 7) + 16 (t >> 4) (low half)
    // and that + 8 (high half) of this warp's 32 rows, for bin (t >> 3) & 1 of the MMA's two.
    const int src_lo = (lane & 7) + 16 * (lane >> 4);
    const int src_hi = src_lo + 8;
    const uint32_t half_shift = 16u * ((lane >> 3) & 1);
    const uint32_t lane_base = tmem_base + ((uint32_t)(quad * 32) << 16);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int64_t mp;
    int nt;
    // this row's codes, loaded one tile ahead so a tile boundary does not wait on L2 (volatile
    // loads: the compiler may not sink them to their first use at the next tile)
    auto load_codes = [&](int64_t mp_, uint4 (&u)[5]) {
      const int64_t f_ = (2 * mp_ + rank) * BM + r;
      if (f_ < F) {
        const uint4 *src = reinterpret_cast<const uint4 *>(codes + f_ * kMel);
#pragma unroll
        for (int q = 0; q < 5; ++q)
          asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(u[q].x), "=r"(u[q].y), "=r"(u[q].z), "=r"(u[q].w)
                       : "l"(src + q));
      } else {
#pragma unroll
        for (int q = 0; q < 5; ++q) u[q] = make_uint4(0u, 0u, 0u, 0u);
      }
    };
    uint4 next[5];
    if (tile(0, mp, nt)) load_codes(mp, next);
    for (int64_t i = 0; ok && tile(i, mp, nt); ++i) {
      const int64_t f = (2 * mp + rank) * BM + r;
      const bool valid = f < F;
      uint32_t cw[20];
#pragma unroll
      for (int q = 0; q < 5; ++q) {
        cw[4 * q] = next[q].x; cw[4 * q + 1] = next[q].y; cw[4 * q + 2] = next[q].z; cw[4 * q + 3] = next[q].w;
      }
      {
        int64_t mp2;
        int nt2;
        if (tile(i + 1, mp2, nt2)) load_codes(mp2, next);
      }
      if (valid) {
        uint32_t bad = 0;
#pragma unroll
        for (int q = 0; q < 20; ++q) bad |= cw[q] & 0xF0F0F0F0u;
        if (bad) record_error(err, DMEL_DEVERR_CODE_RANGE);
      }
      const uint4 *atab = reinterpret_cast<const uint4 *>(smem + OFF_ATAB);
      const uint32_t *mtab = reinterpret_cast<const uint32_t *>(smem + OFF_MTAB);
#pragma unroll
      for (int kb = 0; kb < KBLOCKS; ++kb) {
        // the stage's one-hot rows and metadata are built before waiting for the slot (the wait
        // is on the stage three back; building them is off that critical loop)
        const uint32_t wlo = cw[2 * kb], whi = cw[2 * kb + 1];
        // bin j of the stage: stored bf16 8j .. 8j + 7 = columns 4j .. 4j + 3, one 16-byte
        // row of the level table (the 1 in column 4j + (c >> 2), low half when c is even)
        uint32_t av[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t c = ((j < 4 ? wlo : whi) >> (8 * (j & 3))) & 15u;
          const uint4 w = atab[valid ? c : 16u];
          av[4 * j] = w.x;
          av[4 * j + 1] = w.y;
          av[4 * j + 2] = w.z;
          av[4 * j + 3] = w.w;
        }
        uint32_t m[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t w = k < 2 ? wlo : whi;
          const uint32_t h = (w >> (16 * (k & 1))) & 0x0F0Fu;  // levels c0 (bits 0-3), c1 (bits 8-11)
          const uint32_t pk = mtab[(h & 15u) | (h >> 4)];
          const uint32_t lo = __shfl_sync(0xffffffffu, pk, src_lo), hi = __shfl_sync(0xffffffffu, pk, src_hi);
          m[k] = ((lo >> half_shift) & 0xFFFFu) | (((hi >> half_shift) & 0xFFFFu) << 16);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(empty_a(stage), phase ^ 1u, err))) { ok = false; break; }
        tmem_st32(lane_base + a_col(stage), av);
        tmem_st4(lane_base + META_COL + 4u * stage, m[0], m[1], m[2], m[3]);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(in_leader(full_a(stage)));
        if (++stage == STAGES_A) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp >= 6 && warp < 6 + EPI_WARPS) {
    // ------------------------------------------------ epilogue: 32 rows x 96 columns per warp
    const int quad = warp & 3;
    const int half = (warp - 6) >> 2;  // columns [96 half, 96 half + 96) of the tile
    const int r = quad * 32 + lane;
    const int cb = half * EPI_COLS;
    float *ssp = reinterpret_cast<float *>(smem + OFF_EPI);  // [2][128] row sums of the halves
    float *scl = ssp + 2 * BM;                               // [128] row scales
    // staging slab of this warp: 32 rows of NP 16-byte pieces (a 32-column chunk), pieces
    // swizzled so both the row-wise writes and the piece-wise reads are free of bank conflicts
    constexpr int NP = 2 * (int)sizeof(OT);  // 4 (bf16) or 8 (fp32)
    constexpr int RB = 16 * NP;
    uint8_t *slab = smem + OFF_STG + (warp - 6) * 32 * 128;
    auto piece = [](int q, int j) {
      return NP == 8 ? (j ^ (q & 7)) : (j ^ ((q >> 1) & 3));
    };
    bool ok = true;
    int64_t mp;
    int nt;
    for (int64_t i = 0; ok && tile(i, mp, nt); ++i) {
      const uint32_t acc = i & 1, acc_phase = (i >> 1) & 1;
      const int64_t m = 2 * mp + rank;
      const bool live = m < n_m_tiles;  // uniform over the CTA: the pair's second half may hold no frame
      const int n0 = nt * BN;
      const int ncols = D - n0 < BN ? D - n0 : BN;
      float scale = 1.0f;
      const float *gt = gsm;
      if (kMode == kScaled) {
        // while the accumulator fills: the column tile's RMSNorm weights, into the buffer of tile
        // i - 2 (which every epilogue warp finished before the barrier of tile i - 1 let this
        // warp through), and this row's scale; the barrier below publishes the weights
        float *gb = gsm + acc * BN_EPI;
        const int t = (warp - 6) * 32 + lane;
        if (t < BN_EPI) gb[t] = t < ncols ? __bfloat162float(gw[n0 + t]) : 0.0f;
        const int64_t f = m * BM + r;
        scale = live && f < F ? __ldg(partials + f) : 0.0f;
        gt = gb;
      }
      // a tile's MMAs take several microseconds: the epilogue warps poll with sleeps meanwhile
      // (polling without them took issue slots from the A producers: 6 % of the kernel's time)
      if (!sp_epi_barrier_and(mbar_wait_backoff(tfull(acc), acc_phase, err, kBackoffNs))) { ok = false; break; }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * ACC_STRIDE + cb;
      if (kMode == kFused && live) {
        float ss = 0.0f;
#pragma unroll
        for (int c = 0; c < EPI_COLS; c += 32) {
          uint32_t v0[16], v1[16];
          tmem_ld16(tbase + c, v0);
          tmem_ld16(tbase + c + 16, v1);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float a = __uint_as_float(v0[q]), b = __uint_as_float(v1[q]);
            ss = fmaf(a, a, ss);
            ss = fmaf(b, b, ss);
          }
        }
        ssp[half * BM + r] = ss;
        sp_epi_barrier();
        if (half == 0) {
          // columns past D are zero in the accumulator (the table loads fill them with zeros)
          st_relaxed_f32(partials + (m * P + nt) * BM + r, ssp[r] + ssp[BM + r]);
          // the other slices' sums: 32 independent loads per sweep (one L2 round trip), swept
          // again until none is the sentinel; added in slice order
          const float *col = partials + m * P * BM + r;
          float tot = 0.0f;
          uint32_t polls = 0;
          for (int q0 = 0; q0 < P; q0 += 32) {
            uint32_t u[32];
            for (;;) {
#pragma unroll
              for (int j = 0; j < 32; ++j) u[j] = q0 + j < P ? ld_relaxed_u32(col + (q0 + j) * BM) : 0u;
              bool ready = true;
#pragma unroll
              for (int j = 0; j < 32; ++j) ready &= u[j] != kSentinel;
              if (ready) break;
              if (++polls > kMaxPolls) {
                record_error(err, DMEL_DEVERR_WAIT_TIMEOUT);
#pragma unroll
                for (int j = 0; j < 32; ++j) u[j] = u[j] == kSentinel ? 0u : u[j];
                break;
              }
              __nanosleep(32);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) tot += __uint_as_float(u[j]);
          }
          scl[r] = 1.0f / sqrtf(tot / (float)D + eps);
        }
        sp_epi_barrier();
        scale = scl[r];
      }
      if (live) {
        // rows of this warp: frames m * BM + 32 quad + q, q = 0..31; lane q holds row q's
        // destination (-1: no frame or not written)
        const int64_t f_warp = m * BM + quad * 32;
        const int64_t my_row = f_warp + lane < F ? map_row(om, f_warp + lane, half == 0 ? err : nullptr) : -1;
#pragma unroll 1
        for (int c0 = cb; c0 < cb + EPI_COLS && c0 < ncols; c0 += EPI_CHUNK) {
          uint32_t v[2][16];
          tmem_ld16(tbase + (c0 - cb), v[0]);
          tmem_ld16(tbase + (c0 - cb) + 16, v[1]);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < NP; ++h) {  // 16-byte piece h of this thread's row
            constexpr int E = 16 / (int)sizeof(OT);
            float x[8];
#pragma unroll
            for (int e = 0; e < E; ++e) {
              const int cc = h * E + e;
              x[e] = __uint_as_float(v[cc >> 4][cc & 15]);
              if (kMode == kFused || kMode == kScaled) x[e] = gt[c0 + cc] * (x[e] * scale);
            }
            *reinterpret_cast<uint4 *>(slab + lane * RB + (piece(lane, h) << 4)) = pack16<OT>(x);
          }
          __syncwarp();
#pragma unroll
          for (int it = 0; it < NP; ++it) {  // 32 / NP rows per instruction
            const int q = it * (32 / NP) + lane / NP, j = lane % NP;
            const uint4 w = *reinterpret_cast<const uint4 *>(slab + q * RB + (piece(q, j) << 4));
            const int col = c0 + j * (16 / (int)sizeof(OT));
            const int64_t rq = om.rows ? __shfl_sync(0xffffffffu, my_row, q) : (f_warp + q < F ? f_warp + q : -1);
            if (rq >= 0 && col < ncols) st_stream16(out + rq * (int64_t)D + n0 + col, w);
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(in_leader(tempty(acc)));
    }
  }

  tc_fence_before();
  cluster_sync();  // every MMA into either CTA's TMEM has completed (the leader waited above)
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- column-stationary sparse product
//
// The same 2:4-sparse one-hot product as embed_sp_kernel, with the table read from memory once
// per launch instead of once per frame tile. Cluster c (a CTA pair) owns the column slice
// [n0_c, n0_c + N_c) of the output: the D / 32 units of 32 columns are spread over the clusters,
// so N_c is 64 or 96 at D = 6144 on 74 clusters. Each CTA keeps its N_c / 2 columns of all 1280
// table rows resident in shared memory (MN-major, 32-byte swizzle atoms of 16 columns, 120 KB at
// most), and every cluster walks every 256-frame pair tile. Per tile the 8 producer warps write
// the compressed one-hot A and its metadata into TMEM (even and odd stages by two warps of each
// lane quarter), the MMA warp issues M = 256, N = N_c, logical K = 32 sparse MMAs from a waiter
// warp's handoffs, and three TMEM accumulators let the MMAs run two tiles ahead of the epilogue.
//
// RMSNorm, without a buffer that grows with the batch: each cluster publishes its rows' sums of
// squares over its slice as 64-bit words (value bits | (pair tile + 1) << 32) in a ring of four
// pair tiles; cluster c reduces rows R = c, c + ncl, ... of each pair tile (one warp per row
// sums the ncl partials in a fixed order) and publishes the total the same way; each CTA then
// reads the totals of its 128 rows. A ring slot is rewritten for tile t + 4 only after every
// cluster has read tile t: a cluster publishes tile t + 4 only after it finished tile t + 3,
// whose totals need every cluster's partial of tile t + 3, which a cluster writes only after it
// finished tile t + 2. The ring is zeroed before each launch, so no tag from an earlier launch
// can match.
namespace cs {
constexpr int BM = 128;                      // frames per CTA (TMEM lanes)
constexpr int MAX_N = 96;                    // columns per cluster, at most
constexpr int UNIT = 32;                     // slice widths are multiples of 32 columns
constexpr int ATOM = 16;                     // 32-byte swizzle atom: 16 columns x 8 rows
constexpr int B_ATOM_BYTES = kRows * 32;     // one resident atom column: 1280 rows x 32 bytes
constexpr int MAX_ATOMS = MAX_N / 2 / ATOM;  // 3 per CTA
constexpr int BKL = 128;                     // logical K per stage: 8 bins
constexpr int KSTAGES = kRows / BKL;         // 10
constexpr int B_BOX = BKL * 32;              // TMA box: 16 columns x 128 rows = 4 KB
constexpr int STAGES_A = 4;                  // A + metadata slots in TMEM
constexpr int N_ACC = 3;
constexpr uint32_t ACC_STRIDE = 128;         // accumulators at TMEM columns 0, 128, 256 (N <= 96 used)
constexpr uint32_t META_COL = 96;            // metadata slots at 96, 100, 104, 108 (after accumulator 0)
constexpr uint32_t A_COL0 = 384;             // A slots at 384, 416, 448, 480 (32 columns each)
constexpr uint32_t TMEM_COLS = 512;
constexpr int PROD_WARPS = 8;                // warps 0..7: lane quarter w & 3, stage parity w >> 2
constexpr int W_EPI0 = 8;                    // warps 8..15: lane quarter w & 3, column half
constexpr int EPI_WARPS = 8;
constexpr int W_TMA = 16, W_MMA = 17, W_WAIT = 18;
constexpr int THREADS = 32 * 19;
constexpr int RING = 4;                      // pair tiles in the RMSNorm exchange ring
constexpr int MAX_CLUSTERS = 128;            // ring sized for up to 256 SMs
constexpr int OFF_B = 0;
constexpr int OFF_BAR = OFF_B + MAX_ATOMS * B_ATOM_BYTES;
constexpr int N_BARS = 2 * STAGES_A + KSTAGES + 2 * N_ACC + 1;
constexpr int OFF_G = OFF_BAR + 256;         // RMSNorm weights of the slice (fp32)
constexpr int OFF_EPI = OFF_G + MAX_N * 4;   // row sums of the two column halves [2][128], scales [128]
constexpr int STG_ROW_MAX = MAX_N / 2 * 4 + 16;  // staging row: up to 48 fp32 + 16 bytes of pad
constexpr int OFF_STG = OFF_EPI + 3 * BM * 4;
constexpr int SMEM_USED = OFF_STG + EPI_WARPS * 32 * STG_ROW_MAX;
constexpr int SMEM_BYTES = SMEM_USED + 1024;
static_assert(KSTAGES * BKL == kRows && KSTAGES % 2 == 0, "stages cover the table; parity splits them");
static_assert(MAX_N <= (int)META_COL && META_COL + 4 * STAGES_A <= ACC_STRIDE && N_ACC * ACC_STRIDE <= A_COL0 &&
                  A_COL0 + 32 * STAGES_A <= TMEM_COLS, "TMEM map");
static_assert(N_BARS * 8 + 16 <= 256, "barrier area");
static_assert(OFF_STG % 16 == 0 && SMEM_BYTES <= 227 * 1024, "shared memory budget");
}  // namespace cs

// Ring bytes of the column-stationary kernel's RMSNorm exchange (partials, then totals).
__host__ __device__ constexpr size_t cs_ring_words(int ncl) {
  return (size_t)cs::RING * 2 * cs::BM * (size_t)ncl + (size_t)cs::RING * 2 * cs::BM;
}

// Named barriers 2..5 ("stage slot j is ready", waiter arrives, MMA warp syncs) and 6..9
// ("stage slot j was issued", MMA warp arrives, waiter syncs), j = stage mod 4.
__device__ __forceinline__ void cs_ready_arrive(int j) { asm volatile("bar.arrive %0, 64;" ::"r"(2 + j) : "memory"); }
__device__ __forceinline__ void cs_ready_sync(int j) { asm volatile("bar.sync %0, 64;" ::"r"(2 + j) : "memory"); }
__device__ __forceinline__ void cs_issued_arrive(int j) { asm volatile("bar.arrive %0, 64;" ::"r"(6 + j) : "memory"); }
__device__ __forceinline__ void cs_issued_sync(int j) { asm volatile("bar.sync %0, 64;" ::"r"(6 + j) : "memory"); }

__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// The 16 metadata bits of one bin at level c (see sp_meta_field), computed without a branch.
__device__ __forceinline__ uint32_t cs_meta16(uint32_t c) {
  return 0x4444u | (((c & 2u) * 5u) << ((c >> 2) << 2));
}

template <typename OT, bool kRms>
__global__ void __launch_bounds__(cs::THREADS, 1)
    embed_cs_kernel(const __grid_constant__ CUtensorMap tmap, const uint8_t *__restrict__ codes, int64_t F, int D,
                    OT *__restrict__ out, OutMap om, unsigned long long *__restrict__ ring,
                    const __nv_bfloat16 *__restrict__ gw, float eps, uint32_t *err) {
  using namespace cs;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = (int)(blockIdx.x >> 1), ncl = (int)(gridDim.x >> 1);
  // this cluster's column slice
  const int U = D / UNIT, uq = U / ncl, ur = U % ncl;
  const int N = UNIT * (uq + (cid < ur ? 1 : 0));
  const int n0 = UNIT * (cid * uq + (cid < ur ? cid : ur));
  const int NH = N / 2;  // columns each CTA holds, and each epilogue warp of a lane quarter stores
  const int64_t n_pm = (F + 2 * BM - 1) / (2 * BM);
  const int64_t n_m_tiles = (F + BM - 1) / BM;

  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  const uint32_t bar0 = smem_addr(bars);
  auto full_a = [&](int s) { return bar0 + 8u * s; };
  auto empty_a = [&](int s) { return bar0 + 8u * (STAGES_A + s); };
  auto bfull = [&](int k) { return bar0 + 8u * (2 * STAGES_A + k); };
  auto tfull = [&](int a) { return bar0 + 8u * (2 * STAGES_A + KSTAGES + a); };
  auto tempty = [&](int a) { return bar0 + 8u * (2 * STAGES_A + KSTAGES + N_ACC + a); };
  const uint32_t done_bar = bar0 + 8u * (2 * STAGES_A + KSTAGES + 2 * N_ACC);
  auto in_leader = [&](uint32_t local_bar) { return mapa_shared(local_bar, 0); };
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_BAR + N_BARS * 8);
  float *gsm = reinterpret_cast<float *>(smem + OFF_G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES_A; ++s) {
      mbar_init(full_a(s), 8);  // the 4 producer warps of a stage parity in each CTA
      mbar_init(empty_a(s), 1);
    }
    for (int k = 0; k < KSTAGES; ++k) mbar_init(bfull(k), 1);  // the leader's expect-tx for both halves
    for (int a = 0; a < N_ACC; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), 2 * EPI_WARPS);  // epilogue warps of both CTAs
    }
    mbar_init(done_bar, 1);
    mbar_fence_init();
  }
  if (kRms && threadIdx.x < N) gsm[threadIdx.x] = __bfloat162float(gw[n0 + threadIdx.x]);
  if (warp == W_MMA) {
    tmem_alloc_pair(smem_addr(tmem_holder), TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == W_TMA && lane == 0) tma_prefetch_desc(&tmap);
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t b_base = smem_addr(smem + OFF_B);

  if (warp == W_TMA) {
    // ------------------------------------------------ this CTA's columns of the whole table, once
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      const int atoms = NH / ATOM;
      const int c0 = n0 + (int)rank * NH;
      for (int k = 0; k < KSTAGES; ++k) {
        if (leader) mbar_arrive_expect_tx(bfull(k), 2u * atoms * B_BOX);
        for (int a = 0; a < atoms; ++a)
          tma_load_2d_pair(b_base + a * B_ATOM_BYTES + k * B_BOX, &tmap, c0 + ATOM * a, k * BKL, in_leader(bfull(k)),
                           pol);
      }
    }
  } else if (warp == W_MMA) {
    // ------------------------------------------------ MMA issue (even CTA): stages come from the waiter
    if (leader) {
      const uint32_t idesc = idesc_bf16_f32(2 * BM, (uint32_t)N, 1) | kIdescSparse;
      int sa = 0;
      for (int64_t i = 0; i < n_pm; ++i) {
        const uint32_t acc = (uint32_t)(i % N_ACC);
        const uint32_t d_tmem = tmem_base + acc * ACC_STRIDE;
        for (int s = 0; s < KSTAGES; ++s) {
          cs_ready_sync(sa);
          if (lane == 0) {
            tc_fence_after();
            const uint32_t a0 = tmem_base + A_COL0 + 32u * sa;
#pragma unroll
            for (int k = 0; k < BKL / 32; ++k) {
              // 32 table rows per MMA (32 x 32 bytes in each atom column); atom columns B_ATOM_BYTES apart
              const uint64_t bdesc =
                  smem_desc(b_base + (uint32_t)(s * BKL + 32 * k) * 32u, (uint32_t)B_ATOM_BYTES, 256u, kSwizzle32B);
              const uint32_t mcol = META_COL + 4u * sa + k;
              tc_mma_sp_pair_ts(d_tmem, a0 + 8u * k, bdesc, idesc | (mcol & 1u), tmem_base + (mcol & ~1u),
                                (s | k) != 0 ? 1u : 0u);
            }
            tc_commit_pair_both(empty_a(sa), 3);
            if (s == KSTAGES - 1) tc_commit_pair_both(tfull(acc), 3);
          }
          __syncwarp();
          cs_issued_arrive(sa);
          sa = (sa + 1) & (STAGES_A - 1);
        }
      }
      if (lane == 0) {
        tc_commit_pair(done_bar);
        mbar_wait(done_bar, 0, err);
      }
    }
  } else if (warp == W_WAIT) {
    // ------------------------------------------------ waits on behalf of the MMA warp (even CTA)
    if (leader) {
      bool ok = true;  // after a timed-out wait: no more waiting, stages still handed over
      uint32_t pmask = 0;
      int64_t n = 0;
      for (int64_t i = 0; i < n_pm; ++i) {
        const uint32_t acc = (uint32_t)(i % N_ACC), acc_phase = (uint32_t)((i / N_ACC) & 1);
        for (int s = 0; s < KSTAGES; ++s, ++n) {
          const int sa = (int)(n & (STAGES_A - 1));
          if (n >= STAGES_A) cs_issued_sync(sa);  // stage n - 4 (same slot) was issued
          if (lane == 0 && ok) {
            if (s == 0) ok = mbar_wait(tempty(acc), acc_phase ^ 1u, err);
            ok = ok && mbar_wait(full_a(sa), (pmask >> sa) & 1u, err);
            if (i == 0) ok = ok && mbar_wait(bfull(s), 0, err);
          }
          pmask ^= 1u << sa;
          __syncwarp();
          cs_ready_arrive(sa);
        }
      }
      for (int64_t q = n > STAGES_A ? n - STAGES_A : 0; q < n; ++q) cs_issued_sync((int)(q & (STAGES_A - 1)));
    }
  } else if (warp < PROD_WARPS) {
    // ------------------------------------------------ compressed one-hot A + metadata into TMEM
    const int quad = warp & 3, par = warp >> 2;  // stages with s % 2 == par
    const int r = quad * 32 + lane;
    const uint32_t lane_base = tmem_base + ((uint32_t)(quad * 32) << 16);
    // metadata lane order: lane t takes rows (t & 7) + 16 (t >> 4) and + 8 for bin (t >> 3) & 1
    // of the MMA's two: one exchange with lane t ^ 8, then a byte permute
    const uint32_t msel = (lane & 8) ? 0x3276u : 0x5410u;
    uint32_t pmask = 0;
    bool ok = true;
    // codes of this row for this warp's stages s = par + 2 j: bytes 8 s .. 8 s + 7
    auto load_codes = [&](int64_t i_, uint2 (&u)[5]) {
      const int64_t f_ = (2 * i_ + rank) * BM + r;
      if (i_ < n_pm && f_ < F) {
        const uint2 *src = reinterpret_cast<const uint2 *>(codes + f_ * kMel) + par;
#pragma unroll
        for (int j = 0; j < 5; ++j) u[j] = __ldg(src + 2 * j);
      } else {
#pragma unroll
        for (int j = 0; j < 5; ++j) u[j] = make_uint2(0u, 0u);
      }
    };
    uint2 next[5];
    load_codes(0, next);
    for (int64_t i = 0; ok && i < n_pm; ++i) {
      const bool valid = (2 * i + rank) * BM + r < F;
      uint2 cw[5];
#pragma unroll
      for (int j = 0; j < 5; ++j) cw[j] = next[j];
      load_codes(i + 1, next);
      if (valid) {
        uint32_t bad = 0;
#pragma unroll
        for (int j = 0; j < 5; ++j) bad |= (cw[j].x | cw[j].y) & 0xF0F0F0F0u;
        if (bad) record_error(err, DMEL_DEVERR_CODE_RANGE);
      }
      const uint32_t one_mask = valid ? 0xFFFFFFFFu : 0u;
#pragma unroll
      for (int j = 0; j < 5; ++j) {
        const int s = par + 2 * j;
        const int sa = (int)((i * KSTAGES + s) & (STAGES_A - 1));
        if (!__all_sync(0xffffffffu, mbar_wait(empty_a(sa), ((pmask >> sa) & 1u) ^ 1u, err))) { ok = false; break; }
        pmask ^= 1u << sa;
        // bin b of the stage at level c: stored bf16 8b .. 8b + 7 (columns 4b .. 4b + 3), the 1
        // in column 4b + (c >> 2), low half when c is even
        uint32_t av[32], cc[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          const uint32_t c = ((b < 4 ? cw[j].x : cw[j].y) >> (8 * (b & 3))) & 15u;
          cc[b] = c;
          const uint32_t one = (0x3F80u << ((c & 1u) << 4)) & one_mask;
#pragma unroll
          for (int g = 0; g < 4; ++g) av[4 * b + g] = (c >> 2) == (uint32_t)g ? one : 0u;
        }
        tmem_st32(lane_base + A_COL0 + 32u * sa, av);
        uint32_t m[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t pk = cs_meta16(cc[2 * k]) | (cs_meta16(cc[2 * k + 1]) << 16);
          const uint32_t p = __shfl_xor_sync(0xffffffffu, pk, 8);
          m[k] = __byte_perm(pk, p, msel);
        }
        tmem_st4(lane_base + META_COL + 4u * sa, m[0], m[1], m[2], m[3]);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(in_leader(full_a(sa)));
      }
    }
  } else {
    // ------------------------------------------------ epilogue: 32 rows x NH columns per warp
    const int ew = warp - W_EPI0;
    const int quad = warp & 3, half = ew >> 2;
    const int r = quad * 32 + lane;
    float *ssp = reinterpret_cast<float *>(smem + OFF_EPI);  // [2][128]
    float *scl = ssp + 2 * BM;                               // [128]
    constexpr int OB = (int)sizeof(OT);
    const int row_bytes = NH * OB, stride = row_bytes + 16, pieces = row_bytes / 16;
    uint8_t *stg = smem + OFF_STG + ew * 32 * STG_ROW_MAX;
    unsigned long long *part = ring;                                   // [RING][256][ncl]
    unsigned long long *tot = ring + (size_t)RING * 2 * BM * ncl;      // [RING][256]
    bool ok = true;
    bool gave_up = false;  // a row-sum wait of this thread timed out: results are invalid, stop waiting
    for (int64_t i = 0; ok && i < n_pm; ++i) {
      const uint32_t acc = (uint32_t)(i % N_ACC), acc_phase = (uint32_t)((i / N_ACC) & 1);
      if (!sp_epi_barrier_and(mbar_wait(tfull(acc), acc_phase, err))) { ok = false; break; }
      tc_fence_after();
      const int64_t m = 2 * i + rank;
      const bool live = m < n_m_tiles;  // uniform over the CTA
      const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * ACC_STRIDE + half * NH;
      float scale = 1.0f;
      if (kRms) {
        const unsigned long long tag = (unsigned long long)(i + 1) << 32;
        const int slot = (int)(i % RING);
        if (live) {
          float ss = 0.0f;
          for (int c = 0; c < NH; c += 16) {
            uint32_t v[16];
            tmem_ld16(tbase + c, v);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) ss = fmaf(__uint_as_float(v[q]), __uint_as_float(v[q]), ss);
          }
          ssp[half * BM + r] = ss;
        }
        sp_epi_barrier();
        const int R = (int)rank * BM + r;  // row of the pair tile
        const bool row_ok = live && i * 2 * BM + R < F;
        if (half == 0 && row_ok)
          st_relaxed_u64(part + ((size_t)slot * 2 * BM + R) * ncl + cid,
                         tag | __float_as_uint(ssp[r] + ssp[BM + r]));
        // this cluster's rows of the reduction in this CTA's half: R = cid + ncl k, one per warp
        for (int k = ew; ; k += EPI_WARPS) {
          const int Rr = cid + ncl * k;
          if (Rr >= 2 * BM) break;
          if (Rr / BM != (int)rank) continue;
          if (i * 2 * BM + Rr >= F) break;
          const unsigned long long *src = part + ((size_t)slot * 2 * BM + Rr) * ncl;
          float sum = 0.0f;
          for (int c0 = 0; c0 < ncl; c0 += 32) {
            const int c = c0 + lane;
            unsigned long long v = 0;
            if (c < ncl) {
              uint32_t polls = 0;
              for (;;) {
                v = ld_relaxed_u64(src + c);
                if ((v & 0xFFFFFFFF00000000ull) == tag) break;
                if (gave_up || ++polls > kMaxPolls) {  // after one timeout this thread stops waiting
                  if (!gave_up) record_error(err, DMEL_DEVERR_WAIT_TIMEOUT);
                  gave_up = true;
                  v = 0;
                  break;
                }
                __nanosleep(64);
              }
            }
            sum += __uint_as_float((uint32_t)v);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          if (lane == 0) st_relaxed_u64(tot + (size_t)slot * 2 * BM + Rr, tag | __float_as_uint(sum));
        }
        if (half == 0 && row_ok) {
          uint32_t polls = 0;
          unsigned long long v;
          for (;;) {
            v = ld_relaxed_u64(tot + (size_t)slot * 2 * BM + R);
            if ((v & 0xFFFFFFFF00000000ull) == tag) break;
            if (gave_up || ++polls > kMaxPolls) {
              if (!gave_up) record_error(err, DMEL_DEVERR_WAIT_TIMEOUT);
              gave_up = true;
              break;
            }
            __nanosleep(64);
          }
          scl[r] = 1.0f / sqrtf(__uint_as_float((uint32_t)v) / (float)D + eps);
        }
        sp_epi_barrier();
        scale = scl[r];
      }
      if (live) {
        const int64_t f_warp = m * BM + quad * 32;
        const int64_t my_row = f_warp + lane < F ? map_row(om, f_warp + lane, half == 0 ? err : nullptr) : -1;
        const int cb = half * NH;  // column of the slice where this warp's columns start
        for (int c = 0; c < NH; c += 16) {
          uint32_t v[16];
          tmem_ld16(tbase + c, v);
          tmem_wait_ld();
          float x[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            x[e] = __uint_as_float(v[e]);
            if (kRms) x[e] = gsm[cb + c + e] * (x[e] * scale);
          }
          uint8_t *dst = stg + lane * stride + c * OB;
#pragma unroll
          for (int h = 0; h < 16 * OB / 16; ++h) {
            float x8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x8[e] = x[(h * (16 / OB) + e) & 15];
            *reinterpret_cast<uint4 *>(dst + 16 * h) = pack16<OT>(x8);
          }
        }
        __syncwarp();
        for (int p = lane; p < 32 * pieces; p += 32) {
          const int q = p / pieces, j = p - q * pieces;
          const uint4 w = *reinterpret_cast<const uint4 *>(stg + q * stride + 16 * j);
          const int64_t rq = om.rows ? __shfl_sync(0xffffffffu, my_row, q) : (f_warp + q < F ? f_warp + q : -1);
          if (rq >= 0) st_stream16(out + rq * (int64_t)D + n0 + cb + j * (16 / OB), w);
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(in_leader(tempty(acc)));
    }
  }

  tc_fence_before();
  cluster_sync();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

}  // namespace

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

namespace {

// Tensor map of the bf16 table [1280 x D]: boxes of box_cols columns x box_rows rows, with the
// swizzle whose span is one box row (64 columns: 128 bytes; 32 columns: 64 bytes; 16 columns:
// 32 bytes).
bool make_table_map(CUtensorMap *tmap, const __nv_bfloat16 *table, int D, int box_rows = tc::BK, int box_cols = 64) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)kRows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = box_cols == 16   ? CU_TENSOR_MAP_SWIZZLE_32B
                               : box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = enc(tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16 *>(table), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Scratch of the tensor-core path with RMSNorm: row sums of squares [frame tile][column tile][128]
// and one arrival counter per frame tile.
struct TcScratch {
  float *partials;
  int *counters;
};

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Partial sums are laid out [frame tile][column tile][128]; the streamed sparse kernel's
// 192-column tiles are the most numerous, so the region is sized for them and the 256-column
// kernels use a prefix.
size_t tc_partials_bytes(int64_t F, int D) {
  const size_t m_tiles = (size_t)((F + tc::BM - 1) / tc::BM);
  return round256(m_tiles * (size_t)sp_col_tiles(D) * tc::BM * sizeof(float));
}

size_t tc_scratch_bytes(int64_t F, int D) {
  const size_t m_tiles = (size_t)((F + tc::BM - 1) / tc::BM);
  return tc_partials_bytes(F, D) + round256(m_tiles * sizeof(int));
}

TcScratch tc_scratch(void *ws, int64_t F, int D) {
  uint8_t *p = static_cast<uint8_t *>(ws);
  TcScratch s;
  s.partials = reinterpret_cast<float *>(p);
  s.counters = reinterpret_cast<int *>(p + tc_partials_bytes(F, D));
  return s;
}

// Whether the fused RMSNorm schedule can run: every block of a group of D/256 blocks must be
// resident at once (cooperative launch, one block per SM).
bool fused_possible(int D, int num_sms, int *grid) {
  static std::atomic<int> coop[256];  // 0 unknown, 1 yes, 2 no
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  int c = coop[dev & 255].load(std::memory_order_relaxed);
  if (c == 0) {
    int v = 0;
    c = (cudaDeviceGetAttribute(&v, cudaDevAttrCooperativeLaunch, dev) == cudaSuccess && v) ? 1 : 2;
    coop[dev & 255].store(c, std::memory_order_relaxed);
  }
  const int P = D / tc::BN;
  const int G = num_sms / P;
  *grid = G * P;
  return c == 1 && G >= 1;
}

bool cooperative_enabled();

template <typename OT, int kMode>
cudaError_t launch_tc(const uint8_t *codes, int64_t F, const __nv_bfloat16 *table, int D, OT *out, OutMap om, TcScratch sc,
                      const __nv_bfloat16 *g, float eps, uint32_t *err, int grid, cudaStream_t stream) {
  static std::atomic<bool> attr[256];
  cudaError_t e = set_smem_attr_once(embed_tc_kernel<OT, kMode>, tc::SMEM_BYTES, attr);
  if (e != cudaSuccess) return e;
  CUtensorMap tmap;
  if (!make_table_map(&tmap, table, D)) return cudaErrorInvalidValue;
  if (kMode == kFused) {
    const int64_t m_tiles = (F + tc::BM - 1) / tc::BM;
    if ((e = cudaMemsetAsync(sc.counters, 0, (size_t)m_tiles * sizeof(int), stream)) != cudaSuccess) return e;
    if (cooperative_enabled()) {
      void *args[] = {&tmap, (void *)&codes, (void *)&F, (void *)&D, (void *)&out, (void *)&om, (void *)&sc.partials,
                      (void *)&sc.counters, (void *)&g, (void *)&eps, (void *)&err};
      return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(embed_tc_kernel<OT, kMode>), dim3(grid),
                                         dim3(tc::THREADS), args, tc::SMEM_BYTES, stream);
    }
  }
  embed_tc_kernel<OT, kMode><<<grid, tc::THREADS, tc::SMEM_BYTES, stream>>>(tmap, codes, F, D, out, om,
                                                                             sc.partials, sc.counters, g, eps, err);
  return cudaGetLastError();
}

template <typename TT, typename OT>
cudaError_t launch_simt(const uint8_t *codes, int64_t F, const TT *table, int D, const TT *g, float eps, OT *out,
                        OutMap om, uint32_t *err, int num_sms, cudaStream_t stream) {
  const int smem = g ? D * (int)sizeof(float) : 0;
  static std::atomic<bool> attr[256];
  cudaError_t e = set_smem_attr_once(embed_simt_kernel<TT, OT>, kSimtMaxDim * (int)sizeof(float), attr);
  if (e != cudaSuccess) return e;
  const int64_t cap = (int64_t)num_sms * 8;
  const int grid = (int)(F < cap ? F : cap);
  embed_simt_kernel<TT, OT><<<grid, kSimtThreads, smem, stream>>>(codes, F, table, D, g, eps, out, om, err);
  return cudaGetLastError();
}

template <typename OT>
cudaError_t launch_rescale(OT *out, OutMap om, int64_t F, int D, const __nv_bfloat16 *g, const float *partials,
                           float eps, int num_sms, cudaStream_t stream) {
  const int64_t blocks_needed = (F + 7) / 8;
  const int64_t cap = (int64_t)num_sms * 8;
  const int grid = (int)(blocks_needed < cap ? blocks_needed : cap);
  rms_rescale_kernel<OT><<<grid, 256, 0, stream>>>(out, om, F, D, g, partials, D / tc::BN, eps);
  return cudaGetLastError();
}

// CTA-pair launch (clusters of 2); cooperative when the fused schedule needs every group
// co-resident. Returns cudaErrorNotSupported when the pairs cannot all be resident at once.
template <typename OT, int kMode>
cudaError_t launch_tc2(const uint8_t *codes, int64_t F, const __nv_bfloat16 *table, int D, OT *out, OutMap om, TcScratch sc,
                       const __nv_bfloat16 *g, float eps, uint32_t *err, int clusters, cudaStream_t stream) {
  static std::atomic<bool> attr[256];
  cudaError_t e = set_smem_attr_once(embed_tc2_kernel<OT, kMode>, tc2::SMEM_BYTES, attr);
  if (e != cudaSuccess) return e;
  CUtensorMap tmap;
  if (!make_table_map(&tmap, table, D)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(tc2::THREADS);
  cfg.dynamicSmemBytes = tc2::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeCooperative;
  at[1].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int resident = 0;
  if (cudaOccupancyMaxActiveClusters(&resident, embed_tc2_kernel<OT, kMode>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return cudaErrorNotSupported;
  }
  if (kMode == kFused) {
    if (resident < clusters) return cudaErrorNotSupported;
    cfg.numAttrs = cooperative_enabled() ? 2 : 1;
    const int64_t m_tiles = (F + tc2::BM - 1) / tc2::BM;
    if ((e = cudaMemsetAsync(sc.counters, 0, (size_t)m_tiles * sizeof(int), stream)) != cudaSuccess) return e;
  } else if (resident < 1) {
    return cudaErrorNotSupported;
  }
  return cudaLaunchKernelEx(&cfg, embed_tc2_kernel<OT, kMode>, tmap, codes, F, D, out, om, sc.partials, sc.counters, g, eps,
                            err);
}

// Sparse CTA-pair launch; same contract as launch_tc2. With RMSNorm every cluster must be
// resident (tiles of one frame tile wait for each other).
template <typename OT, int kMode>
cudaError_t launch_sp(const uint8_t *codes, int64_t F, const __nv_bfloat16 *table, int D, OT *out, OutMap om, TcScratch sc,
                      const __nv_bfloat16 *g, float eps, uint32_t *err, int clusters, cudaStream_t stream) {
  static std::atomic<bool> attr[256];
  cudaError_t e = set_smem_attr_once(embed_sp_kernel<OT, kMode>, sp::SMEM_BYTES, attr);
  if (e != cudaSuccess) return e;
  CUtensorMap tmap;
  if (!make_table_map(&tmap, table, D, sp::BKL, sp::B_BOX_COLS)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(sp::THREADS);
  cfg.dynamicSmemBytes = sp::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeCooperative;
  at[1].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int resident = 0;
  if (cudaOccupancyMaxActiveClusters(&resident, embed_sp_kernel<OT, kMode>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return cudaErrorNotSupported;
  }
  if (kMode == kFused) {
    if (resident < clusters) return cudaErrorNotSupported;
    cfg.numAttrs = cooperative_enabled() ? 2 : 1;
    const int64_t m_tiles = (F + sp::BM - 1) / sp::BM;
    const size_t bytes = (size_t)m_tiles * sp_col_tiles(D) * sp::BM * sizeof(float);
    if ((e = cudaMemsetAsync(sc.partials, 0xFF, bytes, stream)) != cudaSuccess) return e;  // all sentinel
  } else if (resident < 1) {
    return cudaErrorNotSupported;
  }
  // kScaled: the dynamic schedule's tile counter was set to 0 by the scale kernels before it
  return cudaLaunchKernelEx(&cfg, embed_sp_kernel<OT, kMode>, tmap, codes, F, D, out, om, sc.partials, sc.counters, g, eps,
                            err);
}

// Clusters the column-stationary kernel runs on: every resident pair, at most one per 32 columns;
// 0 when a slice would be wider than cs::MAX_N (the resident table would not fit).
int cs_clusters(int D, int resident) {
  const int U = D / cs::UNIT;
  int ncl = resident < U ? resident : U;
  if (ncl > cs::MAX_CLUSTERS) ncl = cs::MAX_CLUSTERS;
  if (ncl < 1) return 0;
  const int widest = cs::UNIT * (U / ncl + (U % ncl ? 1 : 0));
  return widest <= cs::MAX_N ? ncl : 0;
}

// Column-stationary launch: one cluster per resident CTA pair (cooperative with RMSNorm, whose
// exchange needs every cluster resident). cudaErrorNotSupported when it cannot take the request.
template <typename OT, bool kRms>
cudaError_t launch_cs(const uint8_t *codes, int64_t F, const __nv_bfloat16 *table, int D, OT *out, OutMap om,
                      unsigned long long *ring, const __nv_bfloat16 *g, float eps, uint32_t *err, int num_sms,
                      cudaStream_t stream) {
  if (D % cs::UNIT != 0) return cudaErrorNotSupported;
  static std::atomic<bool> attr[256];
  cudaError_t e = set_smem_attr_once(embed_cs_kernel<OT, kRms>, cs::SMEM_BYTES, attr);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(cs::THREADS);
  cfg.dynamicSmemBytes = cs::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeCooperative;
  at[1].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(2 * (num_sms / 2));
  int resident = 0;
  if (cudaOccupancyMaxActiveClusters(&resident, embed_cs_kernel<OT, kRms>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return cudaErrorNotSupported;
  }
  if (resident > num_sms / 2) resident = num_sms / 2;
  const int ncl = cs_clusters(D, resident);
  if (ncl == 0) return cudaErrorNotSupported;
  cfg.gridDim = dim3(2 * ncl);
  CUtensorMap tmap;
  if (!make_table_map(&tmap, table, D, cs::BKL, cs::ATOM)) return cudaErrorInvalidValue;
  if (kRms) {
    cfg.numAttrs = cooperative_enabled() ? 2 : 1;
    if ((e = cudaMemsetAsync(ring, 0, cs_ring_words(ncl) * sizeof(unsigned long long), stream)) != cudaSuccess)
      return e;
  }
  return cudaLaunchKernelEx(&cfg, embed_cs_kernel<OT, kRms>, tmap, codes, F, D, out, om, ring, g, eps, err);
}

// Fused kernels are launched cooperatively, which guarantees that every block of a group is
// resident while the group exchanges row sums. DMEL_COOPERATIVE=0 (read once per process)
// launches the same kernel and grid without that attribute, which profilers that cannot replay
// cooperative cluster launches need; the bounded waits then report DMEL_DEVERR_WAIT_TIMEOUT
// rather than stall if other work keeps some blocks off the GPU.
bool cooperative_enabled() {
  static const bool on = [] {
    const char *v = getenv("DMEL_COOPERATIVE");
    return !(v && strcmp(v, "0") == 0);
  }();
  return on;
}

// One-CTA tiles instead of CTA pairs when the environment sets DMEL_EMBED_TILE=single (read
// once per process; for comparisons and tests).
bool pairs_enabled() {
  static const bool on = [] {
    const char *v = getenv("DMEL_EMBED_TILE");
    return !(v && strcmp(v, "single") == 0);
  }();
  return on;
}

// The 2:4-sparse product unless the environment sets DMEL_EMBED_MMA=dense (read once per
// process; for comparisons and tests).
bool sparse_enabled() {
  static const bool on = [] {
    const char *v = getenv("DMEL_EMBED_MMA");
    return !(v && strcmp(v, "dense") == 0);
  }();
  return on;
}

// The column-stationary kernel only when the environment sets DMEL_EMBED_TABLE=resident (read
// once per process). Measured on B200 it is slower than the streamed-table kernel: a 2:4-sparse
// pair MMA (M = 256, logical K = 32) takes about 97 cycles whatever N is up to 128 (116 at
// N = 192, 148 at N = 256), so the 64- and 96-column slices the resident table allows leave the
// tensor pipe half idle.
bool stationary_enabled() {
  static const bool on = [] {
    const char *v = getenv("DMEL_EMBED_TABLE");
    return v && strcmp(v, "resident") == 0;
  }();
  return on;
}

// RMSNorm scales from G = T T^T for calls of at least kGramMinFrames frames (below that, the
// fixed cost of G, ~30 us, outweighs what the exchange of row sums costs the embedding kernel),
// unless the environment sets DMEL_EMBED_NORM=exchange; DMEL_EMBED_NORM=gram takes the G path at
// every size (read once per process; for comparisons and tests). With G prepared for the table
// beforehand, the G path from kPreparedMinFrames frames: below that, the scale pre-pass and the
// extra launches cost about what the exchange does (measured: even between 8,000 and 12,800
// frames, depending on the GPU's MMA rate; 25-35 us gained from 16,384 frames).
int64_t kGramMinFrames = 16384;
int64_t kPreparedMinFrames = 12288;
bool gram_enabled() {
  static const int mode = [] {
    const char *v = getenv("DMEL_EMBED_NORM");
    if (v && strcmp(v, "exchange") == 0) return 0;
    if (v && strcmp(v, "gram") == 0) return 2;
    return 1;
  }();
  if (mode == 2) kGramMinFrames = kPreparedMinFrames = 1;
  return mode != 0;
}

// Tensor-core embedding of F frames: fused RMSNorm when the group schedule fits, else the
// partial-sum kernel followed by rms_rescale_kernel; no RMSNorm: the plain kernel. CTA pairs
// first; one-CTA tiles when pairs are switched off or cannot launch.
template <typename OT>
cudaError_t run_tc(const uint8_t *codes, int64_t F, const __nv_bfloat16 *T, int D, OT *out, OutMap om, const __nv_bfloat16 *g,
                   float eps, void *workspace, uint32_t *err, int num_sms, cudaStream_t stream, int *launches,
                   bool allow_gram, const float *gram_pre) {
  const int P = D / tc::BN;
  const int64_t tiles = ((F + tc::BM - 1) / tc::BM) * P;
  const int plain_grid = (int)(tiles < num_sms ? tiles : num_sms);
  const int64_t pair_tiles = ((F + 2 * tc2::BM - 1) / (2 * tc2::BM)) * P;
  const int max_clusters = num_sms / 2;
  const int plain_clusters = (int)(pair_tiles < max_clusters ? pair_tiles : max_clusters);
  const TcScratch sc = g ? tc_scratch(workspace, F, D) : TcScratch{nullptr, nullptr};
  cudaError_t e;
  if (pairs_enabled() && sparse_enabled() && stationary_enabled()) {
    e = g ? launch_cs<OT, true>(codes, F, T, D, out, om, reinterpret_cast<unsigned long long *>(workspace), g, eps,
                                err, num_sms, stream)
          : launch_cs<OT, false>(codes, F, T, D, out, om, nullptr, nullptr, eps, err, num_sms, stream);
    if (e == cudaSuccess) {
      ++*launches;
      return e;
    }
    (void)cudaGetLastError();  // refused: the streamed-table kernels below
  }
  const int Psp = sp_col_tiles(D);
  const bool use_g = g && gram_enabled() && (gram_pre ? F >= kPreparedMinFrames : allow_gram && F >= kGramMinFrames);
  if (use_g && pairs_enabled() && sparse_enabled() && max_clusters >= 1) {
    // RMSNorm scales from the codes and G = T T^T first (G computed here, or prepared for the table
    // beforehand), then the product on every cluster with no exchange of row sums
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const float *G = gram_pre ? gram_pre : reinterpret_cast<const float *>(ws);
    void *parts = ws + gram_bytes();
    float *scale = reinterpret_cast<float *>(ws + gram_bytes() + norm_scale_bytes(F) - round256((size_t)F * 4));
    int *ctr = reinterpret_cast<int *>(ws + gram_bytes() + norm_scale_bytes(F));  // dynamic tile counter
    int l = 0;
    e = gram_pre ? cudaSuccess : launch_gram(T, D, reinterpret_cast<float *>(ws), err, stream, &l);
    // (the scale kernels zero the tile counter)
    if (e == cudaSuccess) e = launch_norm_scale(codes, F, D, G, eps, parts, scale, ctr, num_sms, stream, &l);
    if (e == cudaSuccess) {
      const int64_t sp_tiles = ((F + 2 * sp::BM - 1) / (2 * sp::BM)) * Psp;
      const int sp_clusters = (int)(sp_tiles < max_clusters ? sp_tiles : max_clusters);
      e = launch_sp<OT, kScaled>(codes, F, T, D, out, om, TcScratch{scale, ctr}, g, eps, err, sp_clusters, stream);
      if (e == cudaSuccess) {
        *launches += l + 1;
        return e;
      }
    }
    if (e != cudaErrorNotSupported) return e;
    (void)cudaGetLastError();  // sparse pairs refused: the exchange kernels below
  }
  if (pairs_enabled() && sparse_enabled() && max_clusters >= Psp) {
    const int64_t sp_tiles = ((F + 2 * sp::BM - 1) / (2 * sp::BM)) * Psp;
    const int sp_clusters = (int)(sp_tiles < max_clusters ? sp_tiles : max_clusters);
    e = g ? launch_sp<OT, kFused>(codes, F, T, D, out, om, sc, g, eps, err, (max_clusters / Psp) * Psp, stream)
          : launch_sp<OT, kPlain>(codes, F, T, D, out, om, sc, nullptr, eps, err, sp_clusters, stream);
    if (e == cudaSuccess) {
      ++*launches;
      return e;
    }
    (void)cudaGetLastError();  // sparse pairs refused: dense kernels below
  }
  if (!g) {
    if (pairs_enabled()) {
      e = launch_tc2<OT, kPlain>(codes, F, T, D, out, om, sc, nullptr, eps, err, plain_clusters, stream);
      if (e == cudaSuccess) {
        ++*launches;
        return e;
      }
      (void)cudaGetLastError();  // pairs refused: one-CTA tiles below
    }
    e = launch_tc<OT, kPlain>(codes, F, T, D, out, om, sc, nullptr, eps, err, plain_grid, stream);
    if (e == cudaSuccess) ++*launches;
    return e;
  }
  if (pairs_enabled() && max_clusters / P >= 1) {
    e = launch_tc2<OT, kFused>(codes, F, T, D, out, om, sc, g, eps, err, (max_clusters / P) * P, stream);
    if (e == cudaSuccess) {
      ++*launches;
      return e;
    }
    (void)cudaGetLastError();  // pairs refused (co-residency or launch attributes): one-CTA tiles below
  }
  int fgrid = 0;
  if (fused_possible(D, num_sms, &fgrid)) {
    e = launch_tc<OT, kFused>(codes, F, T, D, out, om, sc, g, eps, err, fgrid, stream);
    if (e == cudaSuccess) ++*launches;
    if (e != cudaErrorCooperativeLaunchTooLarge) return e;
    (void)cudaGetLastError();  // clear the refused launch; fall through to the two-kernel form
  }
  e = launch_tc<OT, kPartials>(codes, F, T, D, out, om, sc, g, eps, err, plain_grid, stream);
  if (e == cudaSuccess) ++*launches;
  if (e == cudaSuccess) {
    e = launch_rescale(out, om, F, D, g, sc.partials, eps, num_sms, stream);
    if (e == cudaSuccess) ++*launches;
  }
  return e;
}

}  // namespace

// ---------------------------------------------------------------- allocation-free variant

// Fixed scratch for dmel_embed_noalloc: the RMSNorm partial sums of the tensor-core path live
// here instead of in a caller workspace. Every device that loads the library holds these
// 4 MiB until the process exits; all calls share them.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[256] = {nullptr};
}  // namespace

cudaError_t noalloc_scratch(void **ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    // The array's name is only a host-side stand-in; its device address must be looked up,
    // once per device, with that device current.
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return cudaSuccess;
}

// ---------------------------------------------------------------- bounded-wait self test

// One thread waits on an mbarrier whose phase can never complete (count 2, one arrival) with
// the given poll limit: the wait must give up, record DMEL_DEVERR_WAIT_TIMEOUT and return.
__global__ void wait_timeout_kernel(uint32_t polls, uint32_t *err, int *returned) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_addr(&bar);
  mbar_init(b, 2);
  mbar_fence_init();
  mbar_arrive(b);
  bool done = false;
  for (uint32_t i = 0; i < polls && !done; ++i) done = mbar_try_wait(b, 0);
  if (!done) record_error(err, DMEL_DEVERR_WAIT_TIMEOUT);
  *returned = 1;
}

__device__ int g_selftest_returned;

cudaError_t run_wait_timeout_selftest(uint32_t polls, uint32_t *err, int *h_returned) {
  void *d = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&d, g_selftest_returned);
  if (e != cudaSuccess) return e;
  if ((e = cudaMemset(d, 0, sizeof(int))) != cudaSuccess) return e;
  wait_timeout_kernel<<<1, 1>>>(polls, err, static_cast<int *>(d));
  e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(h_returned, d, sizeof(int), cudaMemcpyDeviceToHost);
  return e;
}

bool embed_uses_tensor_cores(dmel_dtype table_dtype, int embed_dim) {
  return table_dtype == DMEL_BF16 && embed_dim > 0 && embed_dim % tc::BN == 0;
}

size_t embed_exchange_workspace_bytes(int64_t n_frames, int embed_dim, dmel_dtype table_dtype, int with_rmsnorm) {
  if (!with_rmsnorm || !embed_uses_tensor_cores(table_dtype, embed_dim) || n_frames <= 0) return 0;
  // the column-stationary kernel's exchange ring, or the streamed-table kernels' partial sums
  const size_t ring = cs_ring_words(cs::MAX_CLUSTERS) * sizeof(unsigned long long);
  const size_t parts = tc_scratch_bytes(n_frames, embed_dim);
  return ring > parts ? ring : parts;
}

size_t embed_workspace_bytes(int64_t n_frames, int embed_dim, dmel_dtype table_dtype, int with_rmsnorm) {
  const size_t ex = embed_exchange_workspace_bytes(n_frames, embed_dim, table_dtype, with_rmsnorm);
  if (ex == 0) return 0;
  // or G, the per-frame partial sums of squares and the scales of the G path, and its tile counter
  const size_t gp = gram_bytes() + norm_scale_bytes(n_frames) + 256;
  return ex > gp ? ex : gp;
}

cudaError_t launch_embed(const uint8_t *codes, int64_t F, const void *table, dmel_dtype table_dtype, int D,
                         const void *rms_weight, float eps, void *out, dmel_dtype out_dtype, void *workspace,
                         uint32_t *err, int num_sms, cudaStream_t stream, int *launches, const int64_t *out_rows,
                         int64_t out_n_rows, bool allow_gram, const float *gram) {
  if (F <= 0) return cudaSuccess;
  const OutMap om{out_rows, out_n_rows};
  cudaError_t e;
  if (embed_uses_tensor_cores(table_dtype, D)) {
    const auto *T = static_cast<const __nv_bfloat16 *>(table);
    const auto *g = static_cast<const __nv_bfloat16 *>(rms_weight);
    if (out_dtype == DMEL_BF16)
      return run_tc(codes, F, T, D, static_cast<__nv_bfloat16 *>(out), om, g, eps, workspace, err, num_sms, stream,
                    launches, allow_gram, gram);
    return run_tc(codes, F, T, D, static_cast<float *>(out), om, g, eps, workspace, err, num_sms, stream, launches,
                  allow_gram, gram);
  }
  if (table_dtype == DMEL_BF16) {
    const auto *T = static_cast<const __nv_bfloat16 *>(table);
    const auto *g = static_cast<const __nv_bfloat16 *>(rms_weight);
    e = out_dtype == DMEL_BF16
            ? launch_simt(codes, F, T, D, g, eps, static_cast<__nv_bfloat16 *>(out), om, err, num_sms, stream)
            : launch_simt(codes, F, T, D, g, eps, static_cast<float *>(out), om, err, num_sms, stream);
  } else {
    const auto *T = static_cast<const float *>(table);
    const auto *g = static_cast<const float *>(rms_weight);
    e = out_dtype == DMEL_BF16
            ? launch_simt(codes, F, T, D, g, eps, static_cast<__nv_bfloat16 *>(out), om, err, num_sms, stream)
            : launch_simt(codes, F, T, D, g, eps, static_cast<float *>(out), om, err, num_sms, stream);
  }
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace dmel
