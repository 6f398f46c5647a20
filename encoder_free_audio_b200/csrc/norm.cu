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
//                   one CTA per 128 x 128 block of the upper block triangle (55 blocks): the
//                   block of bin groups (g, g'), g <= g', 8 bins x 16 levels each way.
//   norm_partials   per 512-frame chunk and group of 5 blocks: each block staged in shared
//                   memory, each frame's 64 (or, on the diagonal, 36) terms looked up and added
//                   in a fixed order; one partial sum per frame and group.
//   norm_finalize   scale_f = 1 / sqrt((sum of the 11 partials, in group order) / D + eps).
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace dmel {
namespace {

// ---------------------------------------------------------------- G = T T^T

namespace gm {
constexpr int BT = 128;                 // block: 128 table rows x 128 table rows
constexpr int BK = 64;                  // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int STAGES = 4;
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
    gram_kernel(const __grid_constant__ CUtensorMap tmap, int D, float *__restrict__ G, uint32_t *err) {
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
  gram_block(blockIdx.x, g, h);
  const int kblocks = D / BK;

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
        tma_load_2d(smem_addr(smem + OFF_A + stage * OP_STAGE), &tmap, kb * BK, g * BT, full(stage), pol);
        tma_load_2d(smem_addr(smem + OFF_B + stage * OP_STAGE), &tmap, kb * BK, h * BT, full(stage), pol);
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

// ---------------------------------------------------------------- per-frame sums of squares

namespace nm {
constexpr int FRAMES = 512;             // frames per CTA
constexpr int THREADS = 256;            // two frames per thread
constexpr int PER_GROUP = 5;            // G blocks per CTA
constexpr int NGROUPS = (gm::BLOCKS + PER_GROUP - 1) / PER_GROUP;  // 11
constexpr int LD = gm::BT + 4;          // staged row stride (floats): 528 bytes, spreads the banks
constexpr int BLK_FLOATS = gm::BT * LD;
constexpr int OFF_CODES = 0;            // uint8 [80][FRAMES], transposed
constexpr int OFF_G = kMel * FRAMES;    // float [2][BT][LD]
constexpr int SMEM_BYTES = OFF_G + 2 * BLK_FLOATS * 4;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(OFF_G % 16 == 0, "16-byte aligned staging");
}  // namespace nm

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all_but_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// G block (g, h) -> shared memory [128][LD], 16-byte copies spread over the CTA.
__device__ __forceinline__ void stage_block(float *dst, const float *__restrict__ G, int q) {
  int g, h;
  gram_block(q, g, h);
  const float *src = G + (size_t)(g * gm::BT) * kRows + h * gm::BT;
  for (int i = threadIdx.x; i < gm::BT * (gm::BT / 4); i += nm::THREADS) {
    const int r = i / (gm::BT / 4), c4 = i % (gm::BT / 4);
    cp_async16(dst + r * nm::LD + 4 * c4, src + (size_t)r * kRows + 4 * c4);
  }
}

__global__ void __launch_bounds__(nm::THREADS, 1)
    norm_partials_kernel(const uint8_t *__restrict__ codes, int64_t F, const float *__restrict__ G,
                         float *__restrict__ partials) {
  using namespace nm;
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t *csm = smem + OFF_CODES;
  float *gbuf = reinterpret_cast<float *>(smem + OFF_G);
  const int64_t f0 = (int64_t)blockIdx.x * FRAMES;
  const int grp = blockIdx.y;
  const int q0 = grp * PER_GROUP;
  const int q1 = q0 + PER_GROUP < gm::BLOCKS ? q0 + PER_GROUP : gm::BLOCKS;

  stage_block(gbuf, G, q0);
  cp_async_commit();
  // this chunk's codes, transposed to [bin][frame] (frames past F read as level 0, never written)
  for (int i = threadIdx.x; i < FRAMES * (kMel / 16); i += THREADS) {
    const int fl = i / (kMel / 16), part = i % (kMel / 16);
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (f0 + fl < F) u = __ldg(reinterpret_cast<const uint4 *>(codes + (f0 + fl) * kMel) + part);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int b = 0; b < 16; ++b) csm[(16 * part + b) * FRAMES + fl] = (uint8_t)((w[b >> 2] >> (8 * (b & 3))) & 15u);
  }
  float acc[2] = {0.0f, 0.0f};
  for (int q = q0; q < q1; ++q) {
    const int buf = (q - q0) & 1;
    if (q + 1 < q1) {
      stage_block(gbuf + (buf ^ 1) * BLK_FLOATS, G, q + 1);
      cp_async_commit();
      cp_async_wait_all_but_one();
    } else {
      cp_async_wait_all();
    }
    __syncthreads();  // block q (and, the first time, the codes) visible to every thread
    const float *blk = gbuf + buf * BLK_FLOATS;
    int g, h;
    gram_block(q, g, h);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int fl = threadIdx.x + e * THREADS;
      int ci[8], cj[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        ci[i] = csm[(8 * g + i) * FRAMES + fl];
        cj[i] = csm[(8 * h + i) * FRAMES + fl];
      }
      float s = 0.0f;
      if (g != h) {
        // bins of two different groups: every pair once in G's upper block, twice in the sum
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) s += blk[(16 * i + ci[i]) * LD + 16 * j + cj[j]];
        s *= 2.0f;
      } else {
        // one group: the 8 diagonal terms once, the 28 pairs i < j twice
        float off = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          s += blk[(16 * i + ci[i]) * LD + 16 * i + ci[i]];
#pragma unroll
          for (int j = i + 1; j < 8; ++j) off += blk[(16 * i + ci[i]) * LD + 16 * j + ci[j]];
        }
        s += 2.0f * off;
      }
      acc[e] += s;
    }
    __syncthreads();  // everyone is done with this buffer before it is refilled
  }
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int64_t f = f0 + threadIdx.x + e * THREADS;
    if (f < F) partials[(size_t)grp * F + f] = acc[e];
  }
}

__global__ void __launch_bounds__(256) norm_finalize_kernel(const float *__restrict__ partials, int64_t F, int D,
                                                            float eps, float *__restrict__ scale) {
  for (int64_t f = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; f < F; f += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.0f;
#pragma unroll
    for (int q = 0; q < nm::NGROUPS; ++q) s += partials[(size_t)q * F + f];
    scale[f] = 1.0f / sqrtf(s / (float)D + eps);
  }
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

size_t gram_bytes() { return round256((size_t)kRows * kRows * sizeof(float)); }

size_t norm_scale_bytes(int64_t F) {
  return round256((size_t)nm::NGROUPS * (size_t)F * sizeof(float)) + round256((size_t)F * sizeof(float));
}

cudaError_t launch_gram(const void *table, int D, float *G, uint32_t *err, cudaStream_t stream, int *launches) {
  if (D % gm::BK != 0) return cudaErrorInvalidValue;
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
  gram_kernel<<<gm::BLOCKS, gm::THREADS, gm::SMEM_BYTES, stream>>>(tmap, D, G, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  ++*launches;
  return cudaSuccess;
}

cudaError_t launch_norm_scale(const uint8_t *codes, int64_t F, int D, const float *G, float eps, void *scratch,
                              float *scale, cudaStream_t stream, int *launches) {
  if (F <= 0) return cudaSuccess;
  static std::atomic<bool> attr[256];
  cudaError_t e = set_smem_attr_once(norm_partials_kernel, nm::SMEM_BYTES, attr);
  if (e != cudaSuccess) return e;
  float *partials = static_cast<float *>(scratch);
  const dim3 grid((unsigned)((F + nm::FRAMES - 1) / nm::FRAMES), nm::NGROUPS);
  norm_partials_kernel<<<grid, nm::THREADS, nm::SMEM_BYTES, stream>>>(codes, F, G, partials);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  ++*launches;
  const int64_t blocks = (F + 255) / 256;
  norm_finalize_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, stream>>>(partials, F, D, eps, scale);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  ++*launches;
  return cudaSuccess;
}

// Host evaluation of the same per-frame formula (diagnostic): sum of squares of the frame with
// codes c[80] from G [1280 x 1280] (row-major, upper blocks filled), in the kernel's order.
double norm_sumsq_host(const uint8_t *c, const float *G) {
  float acc = 0.0f;
  for (int grp = 0; grp < nm::NGROUPS; ++grp) {
    float part = 0.0f;
    for (int q = grp * nm::PER_GROUP; q < (grp + 1) * nm::PER_GROUP && q < gm::BLOCKS; ++q) {
      int g, h;
      gram_block(q, g, h);
      auto at = [&](int bi, int bj) {
        return G[(size_t)(16 * bi + c[bi]) * kRows + 16 * bj + c[bj]];
      };
      float s = 0.0f;
      if (g != h) {
        for (int i = 0; i < 8; ++i)
          for (int j = 0; j < 8; ++j) s += at(8 * g + i, 8 * h + j);
        s *= 2.0f;
      } else {
        float off = 0.0f;
        for (int i = 0; i < 8; ++i) {
          s += at(8 * g + i, 8 * g + i);
          for (int j = i + 1; j < 8; ++j) off += at(8 * g + i, 8 * g + j);
        }
        s += 2.0f * off;
      }
      part += s;
    }
    acc += part;
  }
  return (double)acc;
}

}  // namespace dmel
