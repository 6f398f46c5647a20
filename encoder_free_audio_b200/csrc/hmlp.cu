// The hierarchical MLP patchifier of the vision path ("Inside Inkling: Audio Design", Part 1 ·
// Modeling: a 4-layer hMLP over 40x40 patches; "Why Thinking Machines Built Inkling Without a
// Vision Encoder": linear layers progressively merge pixels into one embedding per patch).
// Stage 1 maps every 5x5 pixel block (75 values, row / column / channel order) to d1 features;
// stages 2-4 map every 2x2 group of the previous stage's grid (four vectors concatenated in
// top-left, top-right, bottom-left, bottom-right order) to d2, d3 and finally dim features.
// Bias, LayerNorm (eps 1e-6) and GELU follow stages 1-3, bias alone stage 4; every stage's
// output is stored in bf16.
//
// Within a patch the blocks are kept in Morton (quad-tree) order, so the four children of a
// 2x2 group are four consecutive rows and every merge is the previous stage's output read as
// [rows / 4 x 4 d]: no data moves between stages. Stage 1 runs as one tcgen05 kernel (pixel
// gather, K = 80 product, LayerNorm and GELU in its epilogue) when d1 is a multiple of 256 up to
// 1536, else as a gather, this file's GEMM and a row kernel; stages 2-4 run this file's tcgen05
// GEMM (bf16 x bf16 -> fp32, CTA pairs), whose epilogue adds the bias and, for stages 2 and 3,
// the rows' per-tile statistics for the one-pass LayerNorm / GELU / rounding row kernel that
// follows; stage 4 rounds to bf16 in the epilogue itself.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace dmel {
namespace {

constexpr int kPatch = 40;
constexpr int kBlocks = 64;   // 5x5 blocks per patch (8 x 8)
constexpr int kK1 = 75;       // values per block
constexpr int kK1Pad = 80;    // row stride of the gathered blocks (16-byte rows)

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

// GELU(u) = u * Phi(u), Phi the standard normal distribution function, with
// Phi(u) = 1 - erfc(u / sqrt 2) / 2 for u >= 0 and erfc(|u| / sqrt 2) / 2 for u < 0, and erfc(z)
// for z >= 0 from Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.26
// (Hastings): erfc(z) = (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-z^2), t = 1 / (1 + p z),
// absolute error at most 1.5e-7. One reciprocal and one exp2 on the special-function unit.
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// With h = erfc(|u| / sqrt 2) / 2, GELU(u) = max(u, 0) - |u| h for either sign of u; the 1/2
// is folded into the coefficients and 1/sqrt 2 into p.
__device__ __forceinline__ float gelu_erf(float u) {
  constexpr float kPr = 0.3275911f * 0.70710678118654752f;  // p / sqrt 2: t = 1 / (1 + p |u| / sqrt 2)
  constexpr float kH1 = 0.5f * 0.254829592f, kH2 = 0.5f * -0.284496736f, kH3 = 0.5f * 1.421413741f,
                  kH4 = 0.5f * -1.453152027f, kH5 = 0.5f * 1.061405429f;
  constexpr float kNegHalfLog2e = -0.72134752044448170f;  // exp(-u^2 / 2) = 2^(u^2 * this)
  const float t = rcp_approx(fmaf(kPr, fabsf(u), 1.0f));
  const float poly = t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, kH5, kH4), kH3), kH2), kH1);
  const float h = poly * ex2_approx(u * (u * kNegHalfLog2e));
  return fmaf(-fabsf(u), h, fmaxf(u, 0.0f));
}

// One warp per row of d fp32 values that already include the bias, with the row's mean and sum of
// squared deviations per column tile of bn values from the GEMM epilogue (n_tn tiles, the last
// one possibly partial): merged in tile order (Chan et al.'s pairwise update), then LayerNorm with
// gain / shift and GELU, rounded to bf16, in one pass over the row.
__global__ void __launch_bounds__(256) hmlp_row_kernel(const float *__restrict__ in, const float2 *__restrict__ stats,
                                                       int n_tn, int bn, int64_t rows, int d,
                                                       const float *__restrict__ g, const float *__restrict__ be,
                                                       __nv_bfloat16 *__restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const float *x = in + r * d;
    __nv_bfloat16 *y = out + r * d;
    float n = 0.0f, mean = 0.0f, m2 = 0.0f;
    for (int t = 0; t < n_tn; ++t) {
      const float2 st = stats[r * n_tn + t];
      const float nb = (float)(d - t * bn < bn ? d - t * bn : bn);
      const float nn = n + nb, delta = st.x - mean;
      mean += delta * (nb / nn);
      m2 += st.y + delta * delta * (n * nb / nn);
      n = nn;
    }
    const float rstd = 1.0f / sqrtf(m2 / (float)d + 1e-6f);
    for (int j = 4 * lane; j < d; j += 128) {
      const float4 v = *reinterpret_cast<const float4 *>(x + j);
      const float4 gg = *reinterpret_cast<const float4 *>(g + j), bb = *reinterpret_cast<const float4 *>(be + j);
      const float t[4] = {v.x, v.y, v.z, v.w}, gv[4] = {gg.x, gg.y, gg.z, gg.w}, bv[4] = {bb.x, bb.y, bb.z, bb.w};
      float o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) o[k] = gelu_erf((t[k] - mean) * rstd * gv[k] + bv[k]);
      __nv_bfloat162 lo = __floats2bfloat162_rn(o[0], o[1]), hi = __floats2bfloat162_rn(o[2], o[3]);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t *>(&lo);
      pk.y = *reinterpret_cast<uint32_t *>(&hi);
      *reinterpret_cast<uint2 *>(y + j) = pk;
    }
  }
}

// Debug: y = GELU(x) with the kernels' formula, one thread per value.
__global__ void hmlp_gelu_kernel(const float *__restrict__ x, float *__restrict__ y, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    y[i] = gelu_erf(x[i]);
}

// ---------------------------------------------------------------- stage 1, fused (tcgen05)
//
// One tile is two patches = 128 pixel blocks (TMEM lanes). Four gather warps copy the tile's
// pixels (two patches of 40 rows x 240 bytes) into shared memory and build the 128 x 80 bf16
// operand A there (K-major, 128-byte swizzle; values 64..79 in a second K block). A TMA warp
// streams W1 (padded to 80 rows) in chunks of 256 columns; one thread issues the
// 128 x 256 x 80 products into a double-buffered TMEM accumulator. The LayerNorm needs the
// whole row of d1 sums, which does not fit in TMEM, so each tile runs its d1 / 256 chunks
// twice: the first pass gives the row statistics (mean and sum of squared deviations per
// 32 values, merged pairwise), the second recomputes the same sums and writes
// bf16(GELU(LayerNorm(x + b1))), each warp's 32 x 32 box staged in shared memory and stored
// with a TMA bulk-tensor store. The product is tiny (K = 80), so the second pass costs far
// less than storing and re-reading the fp32 sums.
namespace s1 {
constexpr int BM = 128;                 // pixel blocks per tile (two patches)
constexpr int BN = 256;                 // columns per accumulator job
constexpr int KP = 80;                  // K: 75 values + 5 zeros
constexpr int A_KB = BM * 128;          // one 64-wide K block of A: 128 rows x 128 B
constexpr int A_STAGE = 2 * A_KB;       // K blocks 0 (values 0..63) and 1 (values 64..79)
constexpr int A_SLOTS = 2;
constexpr int B_BOX = KP * 128;         // 80 K-rows x 64 columns
constexpr int B_STAGE = (BN / 64) * B_BOX;
constexpr int B_STAGES = 2;
constexpr int STG_ROW = 240;            // bytes of one patch row (40 pixels x 3 x bf16)
constexpr int STG = 2 * kPatch * STG_ROW;
// 8 epilogue warps with 32-column batches measured within 1 % of 16 warps with 16-column
// batches; 16 warps with 32-column batches do not fit the register file without spills.
constexpr int EPI_WARPS = 8;   // EPI_WARPS / 4 per TMEM lane quadrant
constexpr int BATCH = 32;      // columns per TMEM load in the epilogue
constexpr int EPI_PARTS = EPI_WARPS / 4;
constexpr int EPI_COLS = BN / EPI_PARTS;
constexpr int EPI_THREADS = 32 * EPI_WARPS;
constexpr int THREADS = 32 * (6 + EPI_WARPS);
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + A_SLOTS * A_STAGE;
constexpr int OFF_OUT = OFF_B + B_STAGES * B_STAGE;
// output staging: per epilogue warp two buffers of 32 rows x BATCH bf16 (64-byte swizzle),
// written to global memory by TMA bulk stores
constexpr int OUT_BUF = 32 * BATCH * 2;
constexpr int OFF_STG = OFF_OUT + EPI_WARPS * 2 * OUT_BUF;
constexpr int OFF_STAT = OFF_STG + STG;  // [parts][128 rows] (mean, M2)
constexpr int OFF_BAR = OFF_STAT + EPI_PARTS * BM * 8;
constexpr int N_BARS = 2 * B_STAGES + 2 * A_SLOTS + 4 + 1;
constexpr int MAX_D1 = 1536;            // b1, g1, be1 of up to this many columns staged in shared memory
constexpr int OFF_PAR = OFF_BAR + 256;
constexpr int SMEM_USED = OFF_PAR + 3 * MAX_D1 * 4;
constexpr int SMEM_BYTES = SMEM_USED + 1024;
constexpr uint32_t TMEM_COLS = 2 * BN;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(N_BARS * 8 + 4 <= 256, "barrier area");
static_assert((EPI_PARTS == 2 || EPI_PARTS == 4) && EPI_COLS % BATCH == 0, "epilogue split");
static_assert(OFF_OUT % 1024 == 0 && OUT_BUF % 512 == 0, "64-byte swizzle atoms of the output staging");
static_assert(B_STAGE % 1024 == 0 && A_KB % 1024 == 0 && OFF_B % 1024 == 0, "swizzle atoms stay 1024-B aligned");
}  // namespace s1

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"n"(s1::EPI_THREADS) : "memory"); }

// Barrier of a named group that also ANDs a flag across it, so the whole group takes the same
// branch after a bounded wait.
template <int kId, int kCount>
__device__ __forceinline__ bool group_and(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(out)
      : "r"((uint32_t)v), "n"(kId), "n"(kCount)
      : "memory");
  return out != 0;
}

__device__ __forceinline__ void gather_bar() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

__device__ __forceinline__ float4 lds4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// TMA bulk tensor store of a 2D box from shared memory (no multicast), and its bulk-group
// bookkeeping: commit, wait until the source may be overwritten (.read) or until done.
__device__ __forceinline__ void tma_store_2d(const void *tmap, int32_t x, int32_t y, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld_batch(uint32_t taddr, float (&x)[s1::BATCH]) {
  static_assert(s1::BATCH == 32, "two 16-column loads");
  uint32_t a[16], b[16];
  tmem_ld16(taddr, a);
  tmem_ld16(taddr + 16, b);
  tmem_wait_ld();
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    x[k] = __uint_as_float(a[k]);
    x[16 + k] = __uint_as_float(b[k]);
  }
}

__global__ void __launch_bounds__(s1::THREADS, 1)
    hmlp_stage1_kernel(const __grid_constant__ CUtensorMap w1map, const __grid_constant__ CUtensorMap omap,
                       const __nv_bfloat16 *__restrict__ img, int H, int W, int64_t P, int d1,
                       const float *__restrict__ b1, const float *__restrict__ g1, const float *__restrict__ be1,
                       uint32_t *err) {
  using namespace s1;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base, as an offset from the shared array (keeps the shared address space)
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_addr(smem + OFF_BAR);
  auto full_b = [&](int s) { return bar0 + 8u * s; };
  auto empty_b = [&](int s) { return bar0 + 8u * (B_STAGES + s); };
  auto full_a = [&](int s) { return bar0 + 8u * (2 * B_STAGES + s); };
  auto empty_a = [&](int s) { return bar0 + 8u * (2 * B_STAGES + A_SLOTS + s); };
  auto tfull = [&](int a) { return bar0 + 8u * (2 * B_STAGES + 2 * A_SLOTS + a); };
  auto tempty = [&](int a) { return bar0 + 8u * (2 * B_STAGES + 2 * A_SLOTS + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (N_BARS - 1);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_BAR + N_BARS * 8);

  const int NC = d1 / BN;                      // column chunks per row
  float *par = reinterpret_cast<float *>(smem + OFF_PAR);  // b1 | g1 | be1
  for (int i = threadIdx.x; i < d1; i += blockDim.x) {
    par[i] = b1[i];
    par[d1 + i] = g1[i];
    par[2 * d1 + i] = be1[i];
  }
  const int64_t n_tiles = (P + 1) / 2;
  const int64_t rows1 = P * kBlocks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < B_STAGES; ++s) {
      mbar_init(full_b(s), 1);
      mbar_init(empty_b(s), 1);
    }
    for (int s = 0; s < A_SLOTS; ++s) {
      mbar_init(full_a(s), 128);
      mbar_init(empty_a(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), EPI_THREADS);
    }
    mbar_init(done_bar, 1);
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&w1map);
    tma_prefetch_desc(&omap);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------ TMA: W1 chunks, 2 NC per tile
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0, pending = 0, pending_phase = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        for (int j = 0; j < 2 * NC; ++j) {
          if (!mbar_wait(empty_b(stage), phase ^ 1u, err)) { ok = false; break; }
          mbar_arrive_expect_tx(full_b(stage), B_STAGE);
          const uint32_t dst = smem_addr(smem + OFF_B + stage * B_STAGE);
          const int c0 = (j % NC) * BN;
#pragma unroll
          for (int q = 0; q < BN / 64; ++q) tma_load_2d(dst + q * B_BOX, &w1map, c0 + 64 * q, 0, full_b(stage), pol);
          pending |= 1u << stage;
          pending_phase = (pending_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == B_STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      for (int s = 0; s < B_STAGES; ++s)
        if (pending & (1u << s)) mbar_wait(full_b(s), (pending_phase >> s) & 1u, err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, 1);
      int stage = 0;
      uint32_t phase = 0, g = 0;
      bool ok = true;
      uint32_t it = 0;
      for (int64_t t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++it) {
        const uint32_t slot = it & 1u;
        if (!mbar_wait(full_a(slot), (it >> 1) & 1u, err)) break;
        const uint32_t a0 = smem_addr(smem + OFF_A + slot * A_STAGE);
        for (int j = 0; j < 2 * NC; ++j, ++g) {
          const uint32_t acc = g & 1u;
          if (!mbar_wait(tempty(acc), ((g >> 1) & 1u) ^ 1u, err) || !mbar_wait(full_b(stage), phase, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b0 = smem_addr(smem + OFF_B + stage * B_STAGE);
#pragma unroll
          for (int k = 0; k < KP / 16; ++k) {
            // A: K-major, 128-byte swizzle, 8-row groups 1024 B apart; K steps of 32 B within a
            // 64-wide block, the fifth step at the start of the second block.
            const uint64_t adesc = smem_desc(k < 4 ? a0 + 32u * k : a0 + A_KB, 16u, 1024u, kSwizzle128B);
            // B: MN-major, 128-byte swizzle; 64-column boxes B_BOX apart, 8 K-rows 1024 B apart,
            // 16 K-rows (2 KB) per step.
            const uint64_t bdesc = smem_desc(b0 + 2048u * k, (uint32_t)B_BOX, 1024u, kSwizzle128B);
            tc_mma_f16(tmem_base + acc * BN, adesc, bdesc, idesc, k > 0 ? 1u : 0u);
          }
          tc_commit(empty_b(stage));
          tc_commit(tfull(acc));
          if (++stage == B_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(empty_a(slot));
      }
      tc_commit(done_bar);
      mbar_wait(done_bar, 0, err);
    }
  } else if (warp < 6) {
    // ------------------------------------------------ pixel gather: row t of A per thread
    const int t = threadIdx.x - 64;
    const int pw = W / kPatch, ph = H / kPatch;
    uint4 *stg = reinterpret_cast<uint4 *>(smem + OFF_STG);
    const __nv_bfloat16 *stg_h = reinterpret_cast<const __nv_bfloat16 *>(smem + OFF_STG);
    uint32_t it = 0;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const uint32_t slot = it & 1u;
      if (!group_and<2, 128>(mbar_wait(empty_a(slot), ((it >> 1) & 1u) ^ 1u, err))) break;
      // two patches x 40 rows x 15 16-byte pieces, coalesced
      for (int idx = t; idx < 2 * kPatch * 15; idx += 128) {
        const int pp = idx / (kPatch * 15), rem = idx % (kPatch * 15);
        const int row = rem / 15, q = rem % 15;
        const int64_t p = 2 * tile + pp;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (p < P) {
          const int64_t im = p / ((int64_t)ph * pw);
          const int pr = (int)((p / pw) % ph), pc = (int)(p % pw);
          const __nv_bfloat16 *src = img + ((im * H + kPatch * pr + row) * (int64_t)W + kPatch * pc) * 3;
          v = __ldg(reinterpret_cast<const uint4 *>(src) + q);
        }
        stg[(pp * kPatch + row) * 15 + q] = v;
      }
      gather_bar();
      {
        const int pp = t >> 6, m = t & 63;
        const __nv_bfloat16 *base = stg_h + (pp * kPatch + 5 * demorton_r(m)) * (STG_ROW / 2) + 15 * demorton_c(m);
        uint8_t *arow = smem + OFF_A + slot * A_STAGE + (t >> 3) * 1024 + (t & 7) * 128;
#pragma unroll
        for (int c = 0; c < KP / 8; ++c) {
          // values 8c .. 8c + 7 of the row (75 and on are zero) as one 16-byte chunk
          uint32_t wv[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int e = 8 * c + 2 * h;
            const float lo = e < 75 ? __bfloat162float(base[(e / 15) * (STG_ROW / 2) + e % 15]) : 0.0f;
            const float hi =
                e + 1 < 75 ? __bfloat162float(base[((e + 1) / 15) * (STG_ROW / 2) + (e + 1) % 15]) : 0.0f;
            wv[h] = pack_bf16(lo, hi);
          }
          const int kb = c >> 3, cc = c & 7;
          *reinterpret_cast<uint4 *>(arow + kb * A_KB + ((cc ^ (t & 7)) << 4)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(full_a(slot));
      gather_bar();  // the staging buffer is free for the next tile
    }
  } else {
    // ------------------------------------------------ epilogue: row r, EPI_COLS columns per job
    // Each warp waits for the accumulator itself; a warp whose wait gave up skips the work but
    // keeps arriving and joining the statistics barrier, so no thread is left at a barrier.
    const int ew = warp - 6;
    const int quad = warp & 3, part = ew >> 2;
    const int r = quad * 32 + lane;
    float2 *stat = reinterpret_cast<float2 *>(smem + OFF_STAT);
    const uint32_t obuf = smem_addr(smem + OFF_OUT + ew * 2 * OUT_BUF);
    const uint32_t par_b = smem_addr(par), par_g = par_b + 4u * d1, par_e = par_b + 8u * d1;
    uint32_t g = 0, n_stored = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
      float n_run = 0.0f, mean_run = 0.0f, m2_run = 0.0f, mean = 0.0f, rstd = 1.0f;
      for (int j = 0; j < 2 * NC; ++j, ++g) {
        const uint32_t acc = g & 1u;
        ok = __all_sync(0xffffffffu, ok && mbar_wait(tfull(acc), (g >> 1) & 1u, err));
        tc_fence_after();
        const uint32_t tb = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * BN + EPI_COLS * part;
        const int col0 = (j % NC) * BN + EPI_COLS * part;
        // the 32 rows of this warp exist (a ragged last tile has one patch: rows 64..127 do not)
        const int64_t row0 = tile * BM + quad * 32;
        if (ok && j < NC) {
          // pass 1: per BATCH values the mean and sum of squared deviations, merged into the run
#pragma unroll 1
          for (int c = 0; c < EPI_COLS / BATCH; ++c) {
            float x[BATCH];
            tmem_ld_batch(tb + BATCH * c, x);
            float s = 0.0f;
#pragma unroll
            for (int k = 0; k < BATCH; k += 4) {
              const float4 b = lds4(par_b + 4u * (col0 + BATCH * c + k));
              x[k] += b.x; x[k + 1] += b.y; x[k + 2] += b.z; x[k + 3] += b.w;
              s += (x[k] + x[k + 1]) + (x[k + 2] + x[k + 3]);
            }
            const float mb = s * (1.0f / BATCH);
            float q = 0.0f;
#pragma unroll
            for (int k = 0; k < BATCH; ++k) {
              const float dv = x[k] - mb;
              q = fmaf(dv, dv, q);
            }
            const float n_new = n_run + (float)BATCH, delta = mb - mean_run;
            mean_run += delta * ((float)BATCH / n_new);
            m2_run += q + delta * delta * (n_run * (float)BATCH / n_new);
            n_run = n_new;
          }
        } else if (ok && row0 < rows1) {
          // pass 2: the same sums again, normalised, GELU, bf16
#pragma unroll 1
          for (int c = 0; c < EPI_COLS / BATCH; ++c) {
            float x[BATCH];
            tmem_ld_batch(tb + BATCH * c, x);
            uint32_t pk[BATCH / 2];
#pragma unroll
            for (int k = 0; k < BATCH; k += 4) {
              const int col = col0 + BATCH * c + k;
              const float4 b = lds4(par_b + 4u * col), gg = lds4(par_g + 4u * col), bb = lds4(par_e + 4u * col);
              const float bv[4] = {b.x, b.y, b.z, b.w}, gv[4] = {gg.x, gg.y, gg.z, gg.w},
                          ev[4] = {bb.x, bb.y, bb.z, bb.w};
              float y[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) y[e] = gelu_erf(fmaf((x[k + e] + bv[e] - mean) * rstd, gv[e], ev[e]));
              pk[k / 2] = pack_bf16(y[0], y[1]);
              pk[k / 2 + 1] = pack_bf16(y[2], y[3]);
            }
            // row r of the warp's 32 x 32 box, 16-byte chunk v at v ^ ((r >> 1) & 3) (64-byte swizzle);
            // the buffer written two batches ago must have been read by its store first
            const uint32_t buf = obuf + (n_stored & 1u) * OUT_BUF;
            if (lane == 0 && n_stored >= 2) bulk_wait_read<1>();
            __syncwarp();
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint32_t a = buf + lane * 64 + ((v ^ ((lane >> 1) & 3)) << 4);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk[4 * v]), "r"(pk[4 * v + 1]),
                           "r"(pk[4 * v + 2]), "r"(pk[4 * v + 3])
                           : "memory");
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&omap, col0 + BATCH * c, (int32_t)row0, buf);
              bulk_commit();
            }
            ++n_stored;
          }
        }
        tc_fence_before();
        mbar_arrive(tempty(acc));
        if (j == NC - 1) {
          // the row's parts (n_run values each), merged pairwise in a fixed order
          stat[part * BM + r] = make_float2(mean_run, m2_run);
          epi_bar();
          float m[EPI_PARTS], q[EPI_PARTS];
#pragma unroll
          for (int a = 0; a < EPI_PARTS; ++a) {
            const float2 v = stat[a * BM + r];
            m[a] = v.x;
            q[a] = v.y;
          }
          float cnt = n_run;
#pragma unroll
          for (int w = 1; w < EPI_PARTS; w *= 2) {
#pragma unroll
            for (int a = 0; a < EPI_PARTS; a += 2 * w) {
              const float d = m[a + w] - m[a];
              m[a] += 0.5f * d;
              q[a] += q[a + w] + d * d * (0.5f * cnt);
            }
            cnt *= 2.0f;
          }
          mean = m[0];
          rstd = 1.0f / sqrtf(q[0] / (float)d1 + 1e-6f);
          epi_bar();  // every thread has read the statistics before the next tile writes them
        }
      }
    }
    if (lane == 0) bulk_wait<0>();  // stores done before the block's shared memory goes away
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- stage GEMMs (tcgen05, CTA pairs)
//
// C [M x N] fp32 = A [M x K] bf16 (row-major, K contiguous) * B [K x N] bf16 (row-major, N
// contiguous), for the merges of stages 2-4 (and stage 1 when it does not run fused). A pair of
// CTAs computes a 256 x 192 tile: each CTA loads its 128 rows of A (K-major, 128-byte swizzle)
// and its 96-column half of B (N-major, 64-byte swizzle) per 64-wide K block by TMA; the even
// CTA's thread issues M = 256, N = 192, K = 16 MMAs into a double-buffered TMEM accumulator of
// both CTAs. Four epilogue warps per CTA move their 32 rows x 192 columns out of TMEM in 32 x 32
// fp32 boxes through shared memory and TMA bulk-tensor stores. Rows past M and columns past N
// (and K past the end) are zero-filled by the loads and clipped by the stores, so any M, N and
// K that are multiples of 8 work.
// What the GEMM's epilogue writes: the fp32 product (kEpiF32); the fp32 product plus the bias and,
// per row and column tile, the mean and sum of squared deviations of those values (kEpiStats: the
// LayerNorm of the row kernel then reads each value once); bf16(product + bias) (kEpiBiasBf16:
// the last stage, which has no LayerNorm).
enum GemmEpi { kEpiF32 = 0, kEpiStats = 1, kEpiBiasBf16 = 2 };

// Tile configuration for pair tiles of 256 x kBN (kBN = 192 or 256): as many K stages as fit
// beside the output staging (one 4 KB box buffer per epilogue warp, two when that costs no stage).
template <int kBN>
struct G2 {
  static constexpr int BM = 128;                      // rows per CTA (256 per pair)
  static constexpr int BN = kBN;                      // columns per pair tile
  static constexpr int BNH = BN / 2;                  // columns of B each CTA loads
  static constexpr int BK = 64;                       // K per stage: one 128-byte row of A
  static constexpr int A_STAGE = BM * BK * 2;         // 16 KB
  static constexpr int B_BOX_COLS = 32;               // 64-byte rows
  static constexpr int B_BOX = B_BOX_COLS * BK * 2;   // 32 columns x 64 K rows = 4 KB
  static constexpr int B_BOXES = BNH / B_BOX_COLS;
  static constexpr int B_STAGE = B_BOXES * B_BOX;
  static constexpr int STAGE = A_STAGE + B_STAGE;
  static constexpr int EPI_WARPS = 4;                 // one per TMEM lane quadrant
  static constexpr int OUT_COLS = 32;                 // fp32 output box: 32 rows x 32 columns (128-byte rows)
  static constexpr int OUT_BUF = 32 * OUT_COLS * 4;   // 4 KB
  static constexpr int BUDGET = 227 * 1024 - 1024 - 256;
  static constexpr int OUT_BUFS =
      (BUDGET - EPI_WARPS * 2 * OUT_BUF) / STAGE == (BUDGET - EPI_WARPS * OUT_BUF) / STAGE ? 2 : 1;
  static constexpr int STAGES = (BUDGET - EPI_WARPS * OUT_BUFS * OUT_BUF) / STAGE;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
  static constexpr int OFF_OUT = OFF_B + STAGES * B_STAGE;
  static constexpr int OFF_BAR = OFF_OUT + EPI_WARPS * OUT_BUFS * OUT_BUF;
  static constexpr int N_BARS = 2 * STAGES + 4 + 1;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
  static constexpr int THREADS = 32 * (2 + EPI_WARPS);  // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
  static constexpr uint32_t ACC_STRIDE = 256;           // accumulators at TMEM columns 0 and 256
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(N_BARS * 8 + 8 <= 256, "barrier area");
  static_assert(A_STAGE % 1024 == 0 && B_STAGE % 1024 == 0 && OFF_OUT % 1024 == 0 && OUT_BUF % 1024 == 0,
                "swizzle atoms stay aligned");
  static_assert(B_BOXES * B_BOX_COLS == BNH && BN <= (int)ACC_STRIDE && STAGES >= 4, "tile split");
};

__device__ __forceinline__ bool g2_tile_at(int64_t i, int64_t n_tiles, int n_tn, int64_t &mp, int &nt) {
  const int64_t t = (int64_t)(blockIdx.x >> 1) + i * (int64_t)(gridDim.x >> 1);
  mp = t / n_tn;  // consecutive clusters share a row block of A (read once into L2)
  nt = (int)(t % n_tn);
  return t < n_tiles;
}

template <int kBN, int kEpi>
__global__ void __launch_bounds__(G2<kBN>::THREADS, 1)
    hmlp_gemm_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                     const __grid_constant__ CUtensorMap cmap, int64_t M, int N, int K, const float *__restrict__ bias,
                     float2 *__restrict__ stats, uint32_t *err) {
  using G = G2<kBN>;
  constexpr int BM = G::BM, BN = G::BN, BNH = G::BNH, BK = G::BK, STAGES = G::STAGES;
  constexpr int A_STAGE = G::A_STAGE, B_STAGE = G::B_STAGE, B_BOX = G::B_BOX, B_BOX_COLS = G::B_BOX_COLS;
  constexpr int B_BOXES = G::B_BOXES, EPI_WARPS = G::EPI_WARPS, OUT_COLS = G::OUT_COLS, OUT_BUF = G::OUT_BUF;
  constexpr int OUT_BUFS = G::OUT_BUFS, OFF_A = G::OFF_A, OFF_B = G::OFF_B, OFF_OUT = G::OFF_OUT;
  constexpr int OFF_BAR = G::OFF_BAR, N_BARS = G::N_BARS;
  constexpr uint32_t ACC_STRIDE = G::ACC_STRIDE, TMEM_COLS = G::TMEM_COLS;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const uint32_t bar0 = smem_addr(smem + OFF_BAR);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_BAR + N_BARS * 8);
  const int n_tn = (N + BN - 1) / BN;
  const int64_t n_tiles = ((M + 2 * BM - 1) / (2 * BM)) * n_tn;
  const int KB = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full(s), 1);   // the even CTA's expect-tx for both CTAs' loads
      mbar_init(empty(s), 1);  // the even CTA's commit, multicast to both
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), 2 * EPI_WARPS);  // the epilogue warps of both CTAs (even CTA's barrier)
    }
    mbar_init(done_bar, 1);
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_addr(tmem_holder), TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&amap);
    tma_prefetch_desc(&bmap);
    tma_prefetch_desc(&cmap);
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------ TMA: this CTA's A rows and B half
    if (lane == 0) {
      const uint64_t keep = policy_evict_last();  // B is re-read by every row block
      int stage = 0;
      uint32_t phase = 0, pending = 0, pending_phase = 0;
      bool ok = true;
      int64_t mp;
      int nt;
      for (int64_t i = 0; ok && g2_tile_at(i, n_tiles, n_tn, mp, nt); ++i) {
        const int32_t row = (int32_t)((2 * mp + rank) * BM);
        const int32_t col = nt * BN + (int32_t)rank * BNH;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(empty(stage), phase ^ 1u, err)) { ok = false; break; }
          const uint32_t fb = mapa_shared(full(stage), 0);
          if (leader) mbar_arrive_expect_tx(full(stage), 2 * (A_STAGE + B_STAGE));
          const uint32_t a_dst = smem_addr(smem + OFF_A + stage * A_STAGE);
          const uint32_t b_dst = smem_addr(smem + OFF_B + stage * B_STAGE);
          tma_load_2d_pair(a_dst, &amap, kb * BK, row, fb, keep);
#pragma unroll
          for (int q = 0; q < B_BOXES; ++q)
            tma_load_2d_pair(b_dst + q * B_BOX, &bmap, col + B_BOX_COLS * q, kb * BK, fb, keep);
          pending |= 1u << stage;
          pending_phase = (pending_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // the even CTA's barriers count every load; it waits for the last ones before leaving
      if (leader)
        for (int s = 0; s < STAGES; ++s)
          if (pending & (1u << s)) mbar_wait(full(s), (pending_phase >> s) & 1u, err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (even CTA)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN, 1);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int64_t mp;
      int nt;
      for (int64_t i = 0; ok && g2_tile_at(i, n_tiles, n_tn, mp, nt); ++i) {
        const uint32_t acc = (uint32_t)(i & 1), use = (uint32_t)(i >> 1);
        if (!mbar_wait(tempty(acc), (use & 1u) ^ 1u, err)) break;
        const uint32_t d = tmem_base + acc * ACC_STRIDE;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(full(stage), phase, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_addr(smem + OFF_A + stage * A_STAGE);
          const uint32_t b0 = smem_addr(smem + OFF_B + stage * B_STAGE);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // A: K-major, 128-byte swizzle, 8-row groups 1024 B apart, 32 B per K step of 16
            const uint64_t adesc = smem_desc(a0 + 32u * k, 16u, 1024u, kSwizzle128B);
            // B: N-major, 64-byte swizzle; 32-column boxes B_BOX apart, 8 K-rows 512 B apart,
            // 16 K-rows (1 KB) per step
            const uint64_t bdesc = smem_desc(b0 + 1024u * k, (uint32_t)B_BOX, 512u, kSwizzle64B);
            tc_mma_f16_pair(d, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit_pair_both(empty(stage), 3);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_both(tfull(acc), 3);
      }
      tc_commit_pair(done_bar);
      mbar_wait(done_bar, 0, err);
    }
  } else {
    // ------------------------------------------------ epilogue: 32 rows x 192 columns per warp
    const int quad = warp & 3;
    const uint32_t obuf = smem_addr(smem + OFF_OUT + (warp - 2) * OUT_BUFS * OUT_BUF);
    uint32_t n_stored = 0;
    bool ok = true;
    int64_t mp;
    int nt;
    for (int64_t i = 0; g2_tile_at(i, n_tiles, n_tn, mp, nt); ++i) {
      const uint32_t acc = (uint32_t)(i & 1), use = (uint32_t)(i >> 1);
      ok = __all_sync(0xffffffffu, ok && mbar_wait(tfull(acc), use & 1u, err));
      tc_fence_after();
      const int64_t row0 = (2 * mp + rank) * BM + 32 * quad;
      const uint32_t tb = tmem_base + ((uint32_t)(32 * quad) << 16) + acc * ACC_STRIDE;
      if (ok && row0 < M) {
        float n_run = 0.0f, mean_run = 0.0f, m2_run = 0.0f;  // kEpiStats: this row over the tile
#pragma unroll 1
        for (int c = 0; c < BN / OUT_COLS; ++c) {
          const int col = nt * BN + OUT_COLS * c;
          if (col >= N) break;
          uint32_t v[2][16];
          tmem_ld16(tb + OUT_COLS * c, v[0]);
          tmem_ld16(tb + OUT_COLS * c + 16, v[1]);
          tmem_wait_ld();
          if (kEpi != kEpiF32) {
            // + bias (columns past N hold zeros from the zero-filled B and stay zero)
#pragma unroll
            for (int k = 0; k < OUT_COLS; ++k) {
              const float b = col + k < N ? __ldg(bias + col + k) : 0.0f;
              v[k >> 4][k & 15] = __float_as_uint(__uint_as_float(v[k >> 4][k & 15]) + b);
            }
          }
          if (kEpi == kEpiStats) {
            // this chunk's mean and sum of squared deviations over its valid columns, merged into
            // the row's run (Chan et al.'s pairwise update)
            const int nv = N - col < OUT_COLS ? N - col : OUT_COLS;
            float sum = 0.0f;
#pragma unroll
            for (int k = 0; k < OUT_COLS; ++k) sum += k < nv ? __uint_as_float(v[k >> 4][k & 15]) : 0.0f;
            const float mb = sum / (float)nv;
            float q = 0.0f;
#pragma unroll
            for (int k = 0; k < OUT_COLS; ++k) {
              const float dv = __uint_as_float(v[k >> 4][k & 15]) - mb;
              q = k < nv ? fmaf(dv, dv, q) : q;
            }
            const float n_new = n_run + (float)nv, delta = mb - mean_run;
            mean_run += delta * ((float)nv / n_new);
            m2_run += q + delta * delta * (n_run * (float)nv / n_new);
            n_run = n_new;
          }
          // the buffer's previous box must have been read by its store first
          const uint32_t buf = obuf + (n_stored % OUT_BUFS) * OUT_BUF;
          if (lane == 0 && n_stored >= (uint32_t)OUT_BUFS) {
            if (OUT_BUFS == 2) bulk_wait_read<1>(); else bulk_wait_read<0>();
          }
          __syncwarp();
          if (kEpi == kEpiBiasBf16) {
            // row `lane` of a 32 x 32 bf16 box: 16-byte chunk j at j ^ ((lane >> 1) & 3) (64-byte swizzle)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t w[4];
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const int k = 8 * j + 2 * h;
                w[h] = pack_bf16(__uint_as_float(v[k >> 4][k & 15]), __uint_as_float(v[(k + 1) >> 4][(k + 1) & 15]));
              }
              const uint32_t a = buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                           "r"(w[3])
                           : "memory");
            }
          } else {
            // row `lane` of a 32 x 32 fp32 box: 16-byte chunk j at j ^ (lane & 7) (128-byte swizzle)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const uint32_t a = buf + lane * 128 + ((j ^ (lane & 7)) << 4);
              const uint32_t *q = &v[j >> 2][4 * (j & 3)];
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(q[0]), "r"(q[1]), "r"(q[2]),
                           "r"(q[3])
                           : "memory");
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&cmap, col, (int32_t)row0, buf);
            bulk_commit();
          }
          ++n_stored;
        }
        if (kEpi == kEpiStats && row0 + lane < M)
          stats[(row0 + lane) * (int64_t)n_tn + nt] = make_float2(mean_run, m2_run);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(mapa_shared(tempty(acc), 0));
    }
    if (lane == 0) bulk_wait<0>();  // stores done before the block's shared memory goes away
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync();  // every MMA into either CTA's TMEM has completed (the even CTA waited above)
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// TMA map of a row-major 2-D bf16 / fp32 array [rows x cols] (row stride `ld` elements), in
// boxes of box_cols x box_rows with the given swizzle.
cudaError_t make_map(CUtensorMap *map, EncodeTiledFn enc, const void *base, CUtensorMapDataType type, size_t es,
                     int64_t rows, int64_t cols, int64_t ld, uint32_t box_cols, uint32_t box_rows,
                     CUtensorMapSwizzle swz) {
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld * (int64_t)es)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(map, type, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  return cudaSuccess;
}

template <int kBN, int kEpi>
cudaError_t launch_gemm_bn(const __nv_bfloat16 *A, int64_t M, int K, int lda, const __nv_bfloat16 *B, int N, void *C,
                           const float *bias, float2 *stats, uint32_t *err, int64_t clusters, cudaStream_t stream) {
  using G = G2<kBN>;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap amap, bmap, cmap;
  cudaError_t e;
  if ((e = make_map(&amap, enc, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, lda, G::BK, G::BM,
                    CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess ||
      (e = make_map(&bmap, enc, B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, N, N, G::B_BOX_COLS, G::BK,
                    CU_TENSOR_MAP_SWIZZLE_64B)) != cudaSuccess)
    return e;
  if (kEpi == kEpiBiasBf16)
    e = make_map(&cmap, enc, C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, N, G::OUT_COLS, 32,
                 CU_TENSOR_MAP_SWIZZLE_64B);
  else
    e = make_map(&cmap, enc, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, M, N, N, G::OUT_COLS, 32,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  static std::atomic<bool> attr[256];
  if ((e = set_smem_attr_once(hmlp_gemm_kernel<kBN, kEpi>, G::SMEM_BYTES, attr)) != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * clusters));
  cfg.blockDim = dim3(G::THREADS);
  cfg.dynamicSmemBytes = G::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, hmlp_gemm_kernel<kBN, kEpi>, amap, bmap, cmap, M, N, K, bias, stats, err);
}

template <int kEpi>
cudaError_t launch_gemm_epi(int bn, const __nv_bfloat16 *A, int64_t M, int K, int lda, const __nv_bfloat16 *B, int N,
                            void *C, const float *bias, float2 *stats, uint32_t *err, int64_t clusters,
                            cudaStream_t stream) {
  return bn == 256 ? launch_gemm_bn<256, kEpi>(A, M, K, lda, B, N, C, bias, stats, err, clusters, stream)
                   : launch_gemm_bn<192, kEpi>(A, M, K, lda, B, N, C, bias, stats, err, clusters, stream);
}

// The tile width launch_gemm takes for an M x N product: 192 or 256 columns, whichever finishes
// its rounds of tiles over the clusters sooner; a 256-column pair MMA takes about 16/15 the time
// of a 192-column one (measured), so the wider tile wins unless it leaves a nearly empty last
// round. Also the number of CTA pairs to launch.
int gemm_tile_width(int64_t M, int N, int num_sms, int64_t *clusters) {
  const int64_t max_clusters = num_sms / 2 > 0 ? num_sms / 2 : 1;
  const int64_t m_pairs = (M + 255) / 256;
  auto rounds = [&](int bn, int64_t &cl) {
    const int64_t tiles = m_pairs * ((N + bn - 1) / bn);
    cl = tiles < max_clusters ? tiles : max_clusters;
    return (tiles + cl - 1) / cl;
  };
  int64_t c192, c256;
  const int64_t r192 = rounds(192, c192), r256 = rounds(256, c256);
  if (16 * r256 < 15 * r192) {
    *clusters = c256;
    return 256;
  }
  *clusters = c192;
  return 192;
}

// Row-major C [M x N] = A [M x K] (row stride lda) * B [K x N], bf16 inputs, fp32 sums, on
// hmlp_gemm_kernel (persistent CTA pairs, one per two SMs at most); the epilogue as `epi` says
// (C fp32 for kEpiF32 and kEpiStats, bf16 for kEpiBiasBf16; stats [M x ceil(N / bn)] for
// kEpiStats, bn the tile width, returned in *bn_out when given).
cudaError_t launch_gemm(const __nv_bfloat16 *A, int64_t M, int K, int lda, const __nv_bfloat16 *B, int N, void *C,
                        int epi, const float *bias, float2 *stats, int *bn_out, uint32_t *err, int num_sms,
                        cudaStream_t stream) {
  if (M <= 0 || N <= 0 || K <= 0) return cudaSuccess;
  if (M > (int64_t)INT32_MAX) return cudaErrorNotSupported;  // TMA row coordinates are 32-bit
  int64_t clusters = 1;
  const int bn = gemm_tile_width(M, N, num_sms, &clusters);
  if (bn_out) *bn_out = bn;
  if (epi == kEpiStats) return launch_gemm_epi<kEpiStats>(bn, A, M, K, lda, B, N, C, bias, stats, err, clusters, stream);
  if (epi == kEpiBiasBf16)
    return launch_gemm_epi<kEpiBiasBf16>(bn, A, M, K, lda, B, N, C, bias, stats, err, clusters, stream);
  return launch_gemm_epi<kEpiF32>(bn, A, M, K, lda, B, N, C, bias, stats, err, clusters, stream);
}

size_t r256(size_t x) { return (x + 255) / 256 * 256; }

struct HmlpLayout {
  size_t a1, h13, h2, f32, stats, w1p, total;
};

// Stage 1 runs fused (hmlp_stage1_kernel) when d1 is a whole number of 256-column chunks, at
// most 1536, and the block rows fit the TMA store's 32-bit row coordinate; otherwise as
// gather + this file's GEMM + row kernel.
bool stage1_fused(int64_t P, const dmel_hmlp_weights &w) {
  return w.d1 % s1::BN == 0 && w.d1 <= s1::MAX_D1 && P * kBlocks <= (int64_t)INT32_MAX;
}

HmlpLayout hmlp_layout(int64_t P, const dmel_hmlp_weights &w) {
  const size_t rows1 = (size_t)P * kBlocks, rows2 = (size_t)P * 16, rows3 = (size_t)P * 4;
  const bool fused = stage1_fused(P, w);
  HmlpLayout L;
  L.a1 = fused ? 0 : r256(rows1 * kK1Pad * 2);
  const size_t h1 = rows1 * (size_t)w.d1, h3 = rows3 * (size_t)w.d3;
  L.h13 = r256((h1 > h3 ? h1 : h3) * 2);
  L.h2 = r256(rows2 * (size_t)w.d2 * 2);
  size_t f = fused ? 0 : rows1 * (size_t)w.d1;
  if (rows2 * (size_t)w.d2 > f) f = rows2 * (size_t)w.d2;
  if (rows3 * (size_t)w.d3 > f) f = rows3 * (size_t)w.d3;
  L.f32 = r256(f * 4);
  // per row and column tile (192 columns at the narrowest) of the stages with LayerNorm
  auto tiles = [](int d) { return (size_t)((d + 191) / 192); };
  size_t st = fused ? 0 : rows1 * tiles(w.d1);
  if (rows2 * tiles(w.d2) > st) st = rows2 * tiles(w.d2);
  if (rows3 * tiles(w.d3) > st) st = rows3 * tiles(w.d3);
  L.stats = r256(st * sizeof(float2));
  L.w1p = r256((size_t)kK1Pad * (size_t)w.d1 * 2);
  L.total = L.a1 + L.h13 + L.h2 + L.f32 + L.stats + L.w1p;
  return L;
}

cudaError_t stage1_smem_attr() {
  static std::atomic<bool> done[256];
  return set_smem_attr_once(hmlp_stage1_kernel, s1::SMEM_BYTES, done);
}

cudaError_t launch_rows(const float *in, const float2 *stats, int bn, int64_t rows, int d, const float *g,
                        const float *be, __nv_bfloat16 *out, int num_sms, cudaStream_t stream) {
  const int64_t blocks = (rows + 7) / 8;
  const int64_t cap = (int64_t)num_sms * 16;
  const unsigned grid = (unsigned)(blocks < cap ? blocks : cap);
  hmlp_row_kernel<<<grid, 256, 0, stream>>>(in, stats, (d + bn - 1) / bn, bn, rows, d, g, be, out);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gelu_debug(const float *x, float *y, int64_t n, int num_sms, cudaStream_t stream) {
  const int64_t blocks = (n + 255) / 256, cap = (int64_t)num_sms * 8;
  hmlp_gelu_kernel<<<(unsigned)(blocks < cap ? blocks : cap), 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_gemm_debug(const void *a, int64_t m, int k, int lda, const void *b, int n, float *c, uint32_t *err,
                              int num_sms, cudaStream_t stream) {
  return launch_gemm(static_cast<const __nv_bfloat16 *>(a), m, k, lda, static_cast<const __nv_bfloat16 *>(b), n, c,
                     kEpiF32, nullptr, nullptr, nullptr, err, num_sms, stream);
}

size_t hmlp_workspace_bytes(int64_t n_patches, const dmel_hmlp_weights &w) {
  return n_patches > 0 ? hmlp_layout(n_patches, w).total : 0;
}

cudaError_t launch_hmlp(const void *images, int n, int H, int W, const dmel_hmlp_weights &w, void *out,
                        void *workspace, uint32_t *err, int num_sms, cudaStream_t stream, int *launches) {
  const int64_t P = (int64_t)n * (H / kPatch) * (W / kPatch);
  if (P <= 0) return cudaSuccess;
  cudaError_t e;
  const HmlpLayout L = hmlp_layout(P, w);
  uint8_t *base = static_cast<uint8_t *>(workspace);
  auto *A1 = reinterpret_cast<__nv_bfloat16 *>(base);
  auto *H13 = reinterpret_cast<__nv_bfloat16 *>(base + L.a1);
  auto *H2 = reinterpret_cast<__nv_bfloat16 *>(base + L.a1 + L.h13);
  auto *F = reinterpret_cast<float *>(base + L.a1 + L.h13 + L.h2);
  auto *S = reinterpret_cast<float2 *>(base + L.a1 + L.h13 + L.h2 + L.f32);
  // W1 padded to 80 rows (5 zero rows) so the stage-1 product has a 16-byte aligned K
  auto *W1 = reinterpret_cast<__nv_bfloat16 *>(base + L.a1 + L.h13 + L.h2 + L.f32 + L.stats);
  if ((e = cudaMemcpyAsync(W1, w.w1, (size_t)kK1 * w.d1 * 2, cudaMemcpyDeviceToDevice, stream)) != cudaSuccess)
    return e;
  if ((e = cudaMemsetAsync(W1 + (size_t)kK1 * w.d1, 0, (size_t)(kK1Pad - kK1) * w.d1 * 2, stream)) != cudaSuccess)
    return e;
  const auto *W2 = static_cast<const __nv_bfloat16 *>(w.w2);
  const auto *W3 = static_cast<const __nv_bfloat16 *>(w.w3);
  const auto *W4 = static_cast<const __nv_bfloat16 *>(w.w4);
  const int64_t rows1 = P * kBlocks, rows2 = P * 16, rows3 = P * 4;
  if (stage1_fused(P, w)) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)w.d1, (cuuint64_t)kK1Pad};
    const cuuint64_t strides[1] = {(cuuint64_t)w.d1 * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kK1Pad};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W1, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    // the stage-1 output [rows1 x d1] bf16, stored in boxes of 32 rows x 32 columns
    CUtensorMap omap;
    const cuuint64_t odims[2] = {(cuuint64_t)w.d1, (cuuint64_t)rows1};
    const cuuint32_t obox[2] = {(cuuint32_t)s1::BATCH, 32};
    if (enc(&omap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H13, odims, strides, obox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    if ((e = stage1_smem_attr()) != cudaSuccess) return e;
    const int64_t tiles = (P + 1) / 2;
    const unsigned grid = (unsigned)(tiles < num_sms ? tiles : num_sms);
    hmlp_stage1_kernel<<<grid, s1::THREADS, s1::SMEM_BYTES, stream>>>(
        map, omap, static_cast<const __nv_bfloat16 *>(images), H, W, P, w.d1, w.b1, w.g1, w.be1, err);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ++*launches;
  } else {
    const int64_t items = P * kBlocks;
    const int64_t cap = (int64_t)num_sms * 16;
    const int64_t blocks = (items + 255) / 256;
    hmlp_gather_kernel<<<(unsigned)(blocks < cap ? blocks : cap), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(images), n, H, W, A1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    int bn = 0;
    if ((e = launch_gemm(A1, rows1, kK1Pad, kK1Pad, W1, w.d1, F, kEpiStats, w.b1, S, &bn, err, num_sms, stream)) !=
        cudaSuccess)
      return e;
    if ((e = launch_rows(F, S, bn, rows1, w.d1, w.g1, w.be1, H13, num_sms, stream)) != cudaSuccess) return e;
    *launches += 3;
  }
  int bn = 0;
  if ((e = launch_gemm(H13, rows2, 4 * w.d1, 4 * w.d1, W2, w.d2, F, kEpiStats, w.b2, S, &bn, err, num_sms, stream)) !=
      cudaSuccess)
    return e;
  if ((e = launch_rows(F, S, bn, rows2, w.d2, w.g2, w.be2, H2, num_sms, stream)) != cudaSuccess) return e;
  if ((e = launch_gemm(H2, rows3, 4 * w.d2, 4 * w.d2, W3, w.d3, F, kEpiStats, w.b3, S, &bn, err, num_sms, stream)) !=
      cudaSuccess)
    return e;
  if ((e = launch_rows(F, S, bn, rows3, w.d3, w.g3, w.be3, H13, num_sms, stream)) != cudaSuccess) return e;
  // the last stage has no LayerNorm: bias and rounding in the GEMM's epilogue, straight into out
  if ((e = launch_gemm(H13, P, 4 * w.d3, 4 * w.d3, W4, w.dim, out, kEpiBiasBf16, w.b4, nullptr, nullptr, err,
                       num_sms, stream)) != cudaSuccess)
    return e;
  *launches += 5;  // stages 2-3: a GEMM and a row kernel each; stage 4: a GEMM
  return cudaSuccess;
}

}  // namespace dmel
