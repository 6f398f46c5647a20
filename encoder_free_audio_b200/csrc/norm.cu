// RMSNorm scales of dMel frames without the frames' vectors ("Inside Inkling: Audio Design",
// Part 1 · Modeling: the 80 rows of a frame are summed, then an optional RMSNorm).
//
// For a frame whose codes select rows r_b = 16 b + c_b of the table T [1280 x D], the vector is
// x = sum_b T[r_b] and its sum of squares is
//     sum_j x_j^2 = sum_b sum_b' G[r_b, r_b'],   G = T T^T  (1280 x 1280, symmetric),
// i.e. the diagonal terms once and every pair b < b' twice. So the scale 1 / sqrt(mean x^2 + eps)
// of every frame follows from its 80 codes and G alone, before (and independently of) the
// embedding's column tiles: the embedding kernel then needs no exchange of row sums between the
// CTAs that own different columns of a row.
//
//   gram_kernel     G = T T^T in fp32 on the tensor cores (bf16 x bf16, fp32 accumulate in TMEM),
//                   one CTA per 128 x 128 block of the upper block triangle (55 blocks: the block
//                   of bin groups (g, g'), g <= g', 8 bins x 16 levels each way) and half of the
//                   D columns (two partial products, 110 CTAs);
//   gram_combine    the two halves added; the 1,280 diagonal entries G[r, r] = sum_j T[r, j]^2
//                   replaced by fp64 sums of the same products: the tensor cores' fp32 accumulation
//                   over thousands of products drifts by ~1e-5 relative, and the diagonal carries
//                   almost all of a frame's sum of squares (80 terms of ~D * var(T) each, against
//                   off-diagonal terms of either sign ~sqrt(D) times smaller).
//   norm_partials   per G block and chunk of 256 E frames (E = 16, or 4, 2, 1 when that would
//                   leave SMs idle): the block staged in shared memory once, each frame's 64 (on the
//                   diagonal 36) terms looked up with eight independent accumulators; one partial
//                   sum per frame and block.
//   norm_finalize   scale_f = 1 / sqrt((sum of the 55 partials, in block order) / D + eps).
#include <cuda.h>
#include <cuda_bf16.h>

#include <vector>

#include "common.cuh"
#include "internal.h"

namespace dmel {
namespace {

// ---------------------------------------------------------------- G = T T^T

namespace gm {
constexpr int BT = 128;                 // block: 128 table rows x 128 table rows
constexpr int BK = 64;                  // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int STAGES = 6;
constexpr int OP_STAGE = BT * BK * 2;   // 16 KB per operand and stage
constexpr int OFF_A = 0;
constexpr int OFF_B = STAGES * OP_STAGE;
constexpr int OFF_BAR = 2 * STAGES * OP_STAGE;
constexpr int N_BARS = 2 * STAGES + 2;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr int THREADS = 192;            // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int GROUPS = kRows / BT;      // 10 bin groups of 8 bins
constexpr int BLOCKS = GROUPS * (GROUPS + 1) / 2;  // 55
constexpr uint32_t TMEM_COLS = 128;
static_assert(N_BARS * 8 + 16 <= 256, "barrier area");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
}  // namespace gm

// Block q of the upper block triangle, row by row: (g, g') with g <= g'.
__host__ __device__ inline void gram_block(int q, int &g, int &h) {
  g = 0;
  while (q >= gm::GROUPS - g) {
    q -= gm::GROUPS - g;
    ++g;
  }
  h = g + q;
}

__global__ void __launch_bounds__(gm::THREADS, 1)
    gram_kernel(const __grid_constant__ CUtensorMap tmap, int D, float *__restrict__ G0, float *__restrict__ G1,
                uint32_t *err) {
  using namespace gm;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  const uint32_t bar0 = smem_addr(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
  const uint32_t tfull = bar0 + 8u * (2 * STAGES);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_BAR + N_BARS * 8);
  int g, h;
  gram_block(blockIdx.x >> 1, g, h);
  const int half = blockIdx.x & 1;  // which half of the D columns (K) this CTA sums
  const int kblocks = D / BK / 2, kb0 = half * kblocks;
  float *__restrict__ G = half ? G1 : G0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(tfull, 1);
    mbar_fence_init();
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
    // ------------------------------------------------ TMA: rows of bin groups g and h, 64 K at a time
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t pending = 0, pending_phase = 0;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait(empty(stage), phase ^ 1u, err)) break;
        mbar_arrive_expect_tx(full(stage), 2 * OP_STAGE);
        tma_load_2d(smem_addr(smem + OFF_A + stage * OP_STAGE), &tmap, (kb0 + kb) * BK, g * BT, full(stage), pol);
        tma_load_2d(smem_addr(smem + OFF_B + stage * OP_STAGE), &tmap, (kb0 + kb) * BK, h * BT, full(stage), pol);
        pending |= 1u << stage;
        pending_phase = (pending_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      for (int s = 0; s < STAGES; ++s)  // every load issued lands before the block exits
        if (pending & (1u << s)) mbar_wait(full(s), (pending_phase >> s) & 1u, err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA: both operands K-major (rows of T)
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BT, BT, 0);
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait(full(stage), phase, err)) break;
        tc_fence_after();
        const uint32_t a0 = smem_addr(smem + OFF_A + stage * OP_STAGE);
        const uint32_t b0 = smem_addr(smem + OFF_B + stage * OP_STAGE);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          // K-major, 128B swizzle: 8-row groups 1024 B apart; K advances 32 B per MMA
          const uint64_t adesc = smem_desc(a0 + 32u * k, 16u, 1024u, kSwizzle128B);
          const uint64_t bdesc = smem_desc(b0 + 32u * k, 16u, 1024u, kSwizzle128B);
          tc_mma_f16(tmem_base, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
        }
        tc_commit(empty(stage));
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      tc_commit(tfull);
    }
  } else {
    // ------------------------------------------------ epilogue: TMEM lanes 32 (warp % 4) .. + 31
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const bool ok = mbar_wait(tfull, 0, err);
    tc_fence_after();
    float *row = G + (size_t)(g * BT + r) * kRows + h * BT;
#pragma unroll 1
    for (int c = 0; c < BT; c += 16) {
      uint32_t v[16];
      tmem_ld16(tmem_base + ((uint32_t)(quad * 32) << 16) + c, v);
      tmem_wait_ld();
      if (ok) {
#pragma unroll
        for (int q = 0; q < 16; q += 4)
          *reinterpret_cast<float4 *>(row + c + q) = make_float4(__uint_as_float(v[q]), __uint_as_float(v[q + 1]),
                                                                 __uint_as_float(v[q + 2]), __uint_as_float(v[q + 3]));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// G0 <- G0 + G1 on the 55 upper blocks (one thread per 4 entries).
__global__ void __launch_bounds__(256) gram_combine_kernel(float *__restrict__ G0, const float *__restrict__ G1) {
  const int per_block = gm::BT * gm::BT / 4;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < gm::BLOCKS * per_block; i += gridDim.x * blockDim.x) {
    int g, h;
    gram_block(i / per_block, g, h);
    const int e = i % per_block, r = e / (gm::BT / 4), c4 = e % (gm::BT / 4);
    const size_t at = (size_t)(g * gm::BT + r) * kRows + h * gm::BT + 4 * c4;
    float4 a = *reinterpret_cast<const float4 *>(G0 + at);
    const float4 b = *reinterpret_cast<const float4 *>(G1 + at);
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
    *reinterpret_cast<float4 *>(G0 + at) = a;
  }
}

// G[r, r] = sum_j T[r, j]^2 in fp64 (each bf16 square is exact; the sum is rounded once): one
// warp per row, each lane a strided share of the D columns, then a fixed reduction tree.
__global__ void __launch_bounds__(256) gram_diag_kernel(const __nv_bfloat16 *__restrict__ T, int D,
                                                         float *__restrict__ G) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= kRows) return;
  const __nv_bfloat16 *row = T + (size_t)r * D;
  double s = 0.0;
  for (int j = 2 * lane; j < D; j += 64) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(row + j);
    const double a = (double)__bfloat162float(v.x), b = (double)__bfloat162float(v.y);
    s += a * a + b * b;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) G[(size_t)r * kRows + r] = (float)s;
}

// ---------------------------------------------------------------- per-frame sums of squares

namespace nm {
constexpr int THREADS = 256;            // frames per CTA: E of them per thread
constexpr int CTAS_PER_SM = 3;
constexpr int LD = gm::BT + 4;          // staged row stride (floats): 528 bytes, spreads the banks
constexpr int BLK_FLOATS = gm::BT * LD;
constexpr int SMEM_BYTES = BLK_FLOATS * 4;  // one G block: 67.6 KB, three CTAs per SM
static_assert(SMEM_BYTES * CTAS_PER_SM <= 227 * 1024, "three CTAs per SM");
}  // namespace nm

// Sum of one frame's terms in G block (g, h) (bin groups g <= h, 8 bins each): ci / cj are the
// row / column offsets 16 i + c and 16 j + c' of the frame's levels in the staged block [128][LD].
// Off the diagonal: all 64 pairs, doubled; on it: the 8 diagonal terms once and the 28 pairs
// i < j twice. Eight accumulators (one per j) keep the additions independent; they are combined
// in a fixed tree.
__host__ __device__ inline float block_terms(const float *blk, const int (&ri)[8], const int (&cj)[8], bool diag) {
  float a[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = 0.0f;
  if (!diag) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) a[j] += blk[ri[i] + cj[j]];
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = i + 1; j < 8; ++j) a[j] += blk[ri[i] + cj[j]];
  }
  float s = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
  s *= 2.0f;
  if (diag) {
    float d[2] = {0.0f, 0.0f};
#pragma unroll
    for (int i = 0; i < 8; ++i) d[i & 1] += blk[ri[i] + cj[i]];
    s += d[0] + d[1];
  }
  return s;
}

// One CTA per (G block q, chunk of THREADS * E frames): the block is staged once, then each
// thread takes E frames THREADS apart, reads the 16 codes of the block's two bin groups straight
// from the codes rows (two 8-byte loads) and writes the frame's partial sum for this block. E is
// a compile-time count, so the loop unrolls and the codes loads run ahead of the lookups.
template <int E>
__global__ void __launch_bounds__(nm::THREADS, nm::CTAS_PER_SM)
    norm_partials_kernel(const uint8_t *__restrict__ codes, int64_t F, const float *__restrict__ G,
                         float *__restrict__ partials) {
  using namespace nm;
  extern __shared__ __align__(16) float blk[];
  const int q = blockIdx.y;
  int g, h;
  gram_block(q, g, h);
  const float *src = G + (size_t)(g * gm::BT) * kRows + h * gm::BT;
  // the block's 16 float4 per thread, all loads in flight before the first store
  constexpr int PER = gm::BT * (gm::BT / 4) / THREADS;
  static_assert(PER * THREADS == gm::BT * (gm::BT / 4), "whole block");
  float4 v[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = threadIdx.x + k * THREADS, r = i / (gm::BT / 4), c4 = i % (gm::BT / 4);
    v[k] = __ldg(reinterpret_cast<const float4 *>(src + (size_t)r * kRows) + c4);
  }
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = threadIdx.x + k * THREADS, r = i / (gm::BT / 4), c4 = i % (gm::BT / 4);
    *reinterpret_cast<float4 *>(blk + r * LD + 4 * c4) = v[k];
  }
  const int64_t f0 = (int64_t)blockIdx.x * (THREADS * E) + threadIdx.x;
  // the codes of this thread's next frame are loaded while the current frame's terms are summed
  auto load = [&](int e, uint2 &ug, uint2 &uh) {
    const int64_t f = f0 + (int64_t)e * THREADS;
    if (e < E && f < F) {
      const uint8_t *row = codes + f * kMel;
      ug = __ldg(reinterpret_cast<const uint2 *>(row + 8 * g));
      uh = __ldg(reinterpret_cast<const uint2 *>(row + 8 * h));
    }
  };
  uint2 ug = make_uint2(0u, 0u), uh = make_uint2(0u, 0u);
  load(0, ug, uh);
  __syncthreads();
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int64_t f = f0 + (int64_t)e * THREADS;
    if (f >= F) break;
    int ri[8], cj[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t cg = ((i < 4 ? ug.x : ug.y) >> (8 * (i & 3))) & 15u;
      const uint32_t ch = ((i < 4 ? uh.x : uh.y) >> (8 * (i & 3))) & 15u;
      ri[i] = (16 * i + (int)cg) * LD;
      cj[i] = 16 * i + (int)ch;
    }
    load(e + 1, ug, uh);
    partials[(size_t)q * F + f] = block_terms(blk, ri, cj, g == h);
  }
}

// scale_f = 1 / sqrt((sum over the 55 blocks, in block order) / D + eps); the 55 loads of a
// frame are all issued before the first addition. Also sets *zero (when given) to 0: the tile
// counter of the product kernel that follows on the stream.
__global__ void __launch_bounds__(256) norm_finalize_kernel(const float *__restrict__ partials, int64_t F, int D,
                                                            float eps, float *__restrict__ scale, int *zero) {
  if (zero && blockIdx.x == 0 && threadIdx.x == 0) *zero = 0;
  for (int64_t f = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; f < F; f += (int64_t)gridDim.x * blockDim.x) {
    float v[gm::BLOCKS];
#pragma unroll
    for (int q = 0; q < gm::BLOCKS; ++q) v[q] = __ldcs(partials + (size_t)q * F + f);
    float s = 0.0f;
#pragma unroll
    for (int q = 0; q < gm::BLOCKS; ++q) s += v[q];
    scale[f] = 1.0f / sqrtf(s / (float)D + eps);
  }
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

size_t gram_bytes() { return 2 * round256((size_t)kRows * kRows * sizeof(float)); }

size_t norm_scale_bytes(int64_t F) {
  return round256((size_t)gm::BLOCKS * (size_t)F * sizeof(float)) + round256((size_t)F * sizeof(float));
}

cudaError_t launch_gram(const void *table, int D, float *G, uint32_t *err, cudaStream_t stream, int *launches) {
  if (D % (2 * gm::BK) != 0) return cudaErrorInvalidValue;
  static std::atomic<bool> attr[256];
  cudaError_t e = set_smem_attr_once(gram_kernel, gm::SMEM_BYTES, attr);
  if (e != cudaSuccess) return e;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  // the table read K-major: inner dimension D (the embedding columns), 1280 rows; boxes of 64 x 128
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)kRows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {(cuuint32_t)gm::BK, (cuuint32_t)gm::BT};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(table), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  float *G1 = G + round256((size_t)kRows * kRows * sizeof(float)) / sizeof(float);
  gram_kernel<<<2 * gm::BLOCKS, gm::THREADS, gm::SMEM_BYTES, stream>>>(tmap, D, G, G1, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  gram_combine_kernel<<<148 * 2, 256, 0, stream>>>(G, G1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  gram_diag_kernel<<<kRows / 8, 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(table), D, G);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  *launches += 3;
  return cudaSuccess;
}

template <int E>
cudaError_t launch_partials(const uint8_t *codes, int64_t F, const float *G, float *partials, cudaStream_t stream) {
  static std::atomic<bool> attr[256];
  cudaError_t e = set_smem_attr_once(norm_partials_kernel<E>, nm::SMEM_BYTES, attr);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((F + nm::THREADS * E - 1) / (nm::THREADS * E)), gm::BLOCKS);
  norm_partials_kernel<E><<<grid, nm::THREADS, nm::SMEM_BYTES, stream>>>(codes, F, G, partials);
  return cudaGetLastError();
}

cudaError_t launch_norm_scale(const uint8_t *codes, int64_t F, int D, const float *G, float eps, void *scratch,
                              float *scale, int *zero, int num_sms, cudaStream_t stream, int *launches) {
  if (F <= 0) return cudaSuccess;
  float *partials = static_cast<float *>(scratch);
  // 16 frames per thread, unless that leaves fewer CTAs than three per SM: then 4, 2 or 1
  const int64_t slots = (int64_t)nm::CTAS_PER_SM * num_sms;
  auto ctas = [&](int64_t e) { return (F + nm::THREADS * e - 1) / (nm::THREADS * e) * gm::BLOCKS; };
  cudaError_t e = ctas(16) >= slots ? launch_partials<16>(codes, F, G, partials, stream)
                  : ctas(4) >= slots ? launch_partials<4>(codes, F, G, partials, stream)
                  : ctas(2) >= slots ? launch_partials<2>(codes, F, G, partials, stream)
                                     : launch_partials<1>(codes, F, G, partials, stream);
  if (e != cudaSuccess) return e;
  ++*launches;
  const int64_t blocks = (F + 255) / 256;
  norm_finalize_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, stream>>>(partials, F, D, eps, scale,
                                                                                       zero);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  ++*launches;
  return cudaSuccess;
}

// Host evaluation of the same per-frame formula (diagnostic): sum of squares of the frame with
// codes c[80] from G [1280 x 1280] (row-major, upper blocks filled), in the kernels' order.
double norm_sumsq_host(const uint8_t *c, const float *G) {
  std::vector<float> blk(nm::BLK_FLOATS);
  float acc = 0.0f;
  for (int q = 0; q < gm::BLOCKS; ++q) {
    int g, h;
    gram_block(q, g, h);
    for (int r = 0; r < gm::BT; ++r)
      for (int k = 0; k < gm::BT; ++k) blk[r * nm::LD + k] = G[(size_t)(g * gm::BT + r) * kRows + h * gm::BT + k];
    int ri[8], cj[8];
    for (int i = 0; i < 8; ++i) {
      ri[i] = (16 * i + c[8 * g + i]) * nm::LD;
      cj[i] = 16 * i + c[8 * h + i];
    }
    acc += block_terms(blk.data(), ri, cj, g == h);
  }
  return (double)acc;
}

}  // namespace dmel
