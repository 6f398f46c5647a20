// dMel codes: framing, periodic Hann window, 1600-point DFT power, 80 HTK mel channels,
// log10, clamp to [-7, 2], 16 equal levels ("Inside Inkling: Audio Design", Part 1 · Modeling;
// the window, DFT size, mel formula, log base/floor and level boundaries are this library's
// readings of what the pages leave open, stated in include/dmel.h).
//
// One warp computes one frame; a warp walks a contiguous run of frames so that consecutive
// frames share half their samples through L1. The DFT runs in fp64, so the power spectrum is
// exact to ~1e-15 relative even in bins ~120 dB below the frame's peak; the mel sums, log10,
// clamp and quantiser then run in fp32, which moves the log-mel value by ~1e-7 at most, far
// inside the 1e-4 band around a level boundary where either neighbouring code is accepted.
//
// Real DFT of 1600 points through one complex DFT of 800 points, z_m = u_{2m} + i u_{2m+1}
// (u = windowed samples). 800 = 25 x 32 with m = 32 j + l and k = k1 + 25 k2:
//   A   lane l (0..31): 25-point DFT over j of z_{32 j + l} (5 x 5, in registers), output k1
//       times W_800^{l k1} -> row k1, column l of the warp's 25 x 32 buffer;
//   C1  the 32-point DFTs over l of each row, as 4 x 8 (l = l0 + 4 l1, k2 = k2a + 8 k2b):
//       100 in-place 8-point DFTs over l1, times W_32^{l0 k2a};
//   C2  200 in-place 4-point DFTs over l0; Z[k1 + 25 (k2a + 8 k2b)] ends in row k1, column
//       k2b + 4 k2a;
//   D   X_k = (Z_k + conj Z_{800-k}) / 2 + W_1600^k (Z_k - conj Z_{800-k}) / (2 i),
//       P_k = |X_k|^2; lane l of round r reads Z at row r, column l and its partner
//       Z_{800-k} at row 25 - r, column 31 - l (both bank-conflict free), so each lane owns
//       two runs of 13 adjacent bins (k = 25 k2 + r ascending and 800 - k descending);
//   E   every bin lies between two adjacent mel points, so it feeds at most two adjacent
//       channels (the falling edge of one triangle, the rising edge of the next); each lane
//       folds its two runs into fp32 channel partials as it computes P_k (no P array), writing a
//       partial when its run crosses into a new channel, then 80 channel sums, log10, clamp,
//       quantise (fp32).
// Each lane reads its 50 samples of a frame straight from global memory (for each j the warp
// reads 64 consecutive samples; half of them were read by the previous frame and sit in L1).
// Every root of unity comes from one fp64 table of W_1600^k, k = 0..800 (W_800 = W_1600^2,
// W_32 = W_1600^50, W_25 = W_1600^64, W^{1600 - k} = conj W^k). The buffer is swizzled so the
// column accesses of A, C1 and C2 are free of shared-memory bank conflicts.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace dmel {
namespace {

// Warps (frames in flight) per block, one block per SM: 12 (168 registers per thread; 14 fit the
// shared memory only without the step-D twiddle table and then spill, which measured slower).
constexpr int kWarpsDefault = 12;
constexpr int kRunLen = 13;        // bins per lane run (rounds r = 0..12 of step D)
constexpr int kMaxFlush = 16;      // channel partials one lane writes per run, at most
constexpr int kMaxSegs = 256;      // channel partials per frame (+ one slot for edge flushes)

// Shared memory of one block: the constant tables once, then one 800-element complex buffer
// per warp (Y, then Z in place, then P in place; the mel partials follow P).
constexpr int kSmW = 0;                                    // double2 [801]: W_1600^k
constexpr int kSmHann = kSmW + 801 * 16;                   // double2 [800]: (w[2m], w[2m+1])
constexpr int kSmTwA = kSmHann + 800 * 16;                 // double2 [25 * 32]: W_800^{l k1}
constexpr int kSmMelW2 = kSmTwA + 800 * 16;                // float2 [2][13][32]: bin weights per lane run
constexpr int kSmTwD = kSmMelW2 + 2 * kRunLen * 32 * 8;    // double2 [2][13][32]: step-D twiddles per lane run
constexpr int kSmSlot = kSmTwD + 2 * kRunLen * 32 * 16;    // ushort [32][2][kMaxFlush]: partial slots
constexpr int kSmFlush = kSmSlot + 32 * 2 * kMaxFlush * 2; // uint [2][32]: run positions of new channels
constexpr int kSmChanSeg = kSmFlush + 64 * 4;              // int [81]: slot range per channel
constexpr int kSmTables = (kSmChanSeg + 84 * 4 + 127) / 128 * 128;
constexpr int kWarpBufBytes = 800 * 16;
__host__ __device__ constexpr int smem_bytes(int warps) { return kSmTables + warps * kWarpBufBytes; }
static_assert(kMaxSegs * 4 <= 2 * 32 * 16, "mel partials fit in rows 0 and 1 of the warp's buffer");
static_assert(smem_bytes(kWarpsDefault) <= 227 * 1024, "shared memory budget");

// Constant tables, filled once per device from host-computed fp64 values.
__device__ double2 d_w1600[kBins];
__device__ double2 d_hann2[800];
__device__ double2 d_twa[800];
__device__ float2 d_melw2[2 * kRunLen * 32];
__device__ double2 d_twd[2 * kRunLen * 32];
__device__ unsigned short d_slot[32 * 2 * kMaxFlush];
__device__ unsigned int d_flush[64];
__device__ int d_chanseg[81];

struct Tables {
  const double2 *w;      // W_1600^k = exp(-2 pi i k / 1600), k = 0..800
  const double2 *hann2;  // periodic Hann pairs (w[2m], w[2m+1]), m = 0..799
  const double2 *twa;    // W_800^{l k1} at [k1 * 32 + l]
  // mel weights of the bins of lane l's runs, run q (0: ascending, 1: descending) round r, at
  // [(q * 13 + r) * 32 + l]: (weight to the lower channel, weight to the channel above it)
  const float2 *melw2;
  // W_1600^k of the bin k of lane l's run q at round r, at [(q * 13 + r) * 32 + l] (a copy of the
  // W table's entry, laid out so the 32 lanes of a round read 32 consecutive entries)
  const double2 *twd;
  const unsigned short *slot;  // partial slots of lane l's run q, in order, at [(l * 2 + q) * kMaxFlush]
  const unsigned int *flush;   // bit r of [q * 32 + l]: the run enters a new channel at round r
  const int *chanseg;          // channel b adds the partials [chanseg[b], chanseg[b + 1])
};

// W_1600^idx for idx in [0, 1600).
__host__ __device__ inline double2 tw(const Tables &T, int idx) {
  if (idx <= 800) return T.w[idx];
  const double2 v = T.w[1600 - idx];
  return make_double2(v.x, -v.y);
}

__host__ __device__ inline void cmul(double &re, double &im, double wr, double wi) {
  const double r = re * wr - im * wi;
  const double i = re * wi + im * wr;
  re = r;
  im = i;
}

// Element (row k1, column c) of a warp's 25 x 32 buffer. The three low bits of the column are
// permuted (bits 3..4 of the column and bit 0 of the row feed in), so that eight lanes of A
// (one row, eight columns), C1 (two rows, columns l0 + 4 l1) and C2 (one row, columns
// l0 + 4 k2a) touch eight different 16-byte bank groups.
__host__ __device__ inline int slot(int k1, int c) {
  const int low = ((c & 3) ^ ((c >> 3) & 3)) | ((((c >> 2) ^ k1) & 1) << 2);
  return k1 * 32 + (c & 24) + low;
}

// Where Z_k sits after step C2: row k % 25, column k2b + 4 k2a with k2 = k / 25.
__host__ __device__ inline int zslot(int k) {
  const int k1 = k % 25, k2 = k / 25;
  return slot(k1, (k2 >> 3) + 4 * (k2 & 7));
}

// 5-point DFT X_k = sum_n x_n W_5^{nk}, W_5 = exp(-2 pi i / 5), of x0..x4 (in place).
__host__ __device__ inline void dft5(double &r0, double &i0, double &r1, double &i1, double &r2, double &i2,
                                     double &r3, double &i3, double &r4, double &i4) {
  const double c1 = 0.30901699437494742410;   // cos(2 pi / 5)
  const double c2 = -0.80901699437494742410;  // cos(4 pi / 5)
  const double s1 = 0.95105651629515357212;   // sin(2 pi / 5)
  const double s2 = 0.58778525229247312917;   // sin(4 pi / 5)
  const double t1r = r1 + r4, t1i = i1 + i4;
  const double t2r = r2 + r3, t2i = i2 + i3;
  const double t3r = r1 - r4, t3i = i1 - i4;
  const double t4r = r2 - r3, t4i = i2 - i3;
  const double ar = r0 + c1 * t1r + c2 * t2r, ai = i0 + c1 * t1i + c2 * t2i;
  const double br = r0 + c2 * t1r + c1 * t2r, bi = i0 + c2 * t1i + c1 * t2i;
  const double ur = s1 * t3r + s2 * t4r, ui = s1 * t3i + s2 * t4i;  // v1 = s1 t3 + s2 t4
  const double vr = s2 * t3r - s1 * t4r, vi = s2 * t3i - s1 * t4i;  // v2 = s2 t3 - s1 t4
  r0 = r0 + t1r + t2r;
  i0 = i0 + t1i + t2i;
  // X1 = a - i v1, X4 = a + i v1, X2 = b - i v2, X3 = b + i v2   (-i v = (v.im, -v.re))
  r1 = ar + ui;
  i1 = ai - ur;
  r4 = ar - ui;
  i4 = ai + ur;
  r2 = br + vi;
  i2 = bi - vr;
  r3 = br - vi;
  i3 = bi + vr;
}

// 8-point DFT X_k = sum_n x_n W_8^{nk} (in place, natural order in and out): radix-2
// decimation in time on the bit-reversed input order.
__host__ __device__ inline void dft8(double (&r)[8], double (&i)[8]) {
  const double h = 0.70710678118654752440;  // cos(pi / 4)
  double ar[8], ai[8];
  const int br[8] = {0, 4, 2, 6, 1, 5, 3, 7};
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    ar[q] = r[br[q]];
    ai[q] = i[br[q]];
  }
  // span 1: W_2^0
#pragma unroll
  for (int q = 0; q < 8; q += 2) {
    const double xr = ar[q + 1], xi = ai[q + 1];
    ar[q + 1] = ar[q] - xr;
    ai[q + 1] = ai[q] - xi;
    ar[q] += xr;
    ai[q] += xi;
  }
  // span 2: W_4^0 = 1, W_4^1 = -i
#pragma unroll
  for (int q = 0; q < 8; q += 4) {
    double xr = ar[q + 2], xi = ai[q + 2];
    ar[q + 2] = ar[q] - xr;
    ai[q + 2] = ai[q] - xi;
    ar[q] += xr;
    ai[q] += xi;
    xr = ai[q + 3];  // (-i) x = (x.im, -x.re)
    xi = -ar[q + 3];
    ar[q + 3] = ar[q + 1] - xr;
    ai[q + 3] = ai[q + 1] - xi;
    ar[q + 1] += xr;
    ai[q + 1] += xi;
  }
  // span 4: W_8^0 = 1, W_8^1 = h (1 - i), W_8^2 = -i, W_8^3 = -h (1 + i)
  {
    double xr, xi;
    xr = ar[4]; xi = ai[4];
    ar[4] = ar[0] - xr; ai[4] = ai[0] - xi; ar[0] += xr; ai[0] += xi;
    xr = h * (ar[5] + ai[5]); xi = h * (ai[5] - ar[5]);
    ar[5] = ar[1] - xr; ai[5] = ai[1] - xi; ar[1] += xr; ai[1] += xi;
    xr = ai[6]; xi = -ar[6];
    ar[6] = ar[2] - xr; ai[6] = ai[2] - xi; ar[2] += xr; ai[2] += xi;
    xr = h * (ai[7] - ar[7]); xi = -h * (ar[7] + ai[7]);
    ar[7] = ar[3] - xr; ai[7] = ai[3] - xi; ar[3] += xr; ai[3] += xi;
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    r[q] = ar[q];
    i[q] = ai[q];
  }
}

// Step A, first half, straight from global memory: lane l reads the samples
// x[800 (t - 1) + 64 j + 2 l] and the next one of frame t (start = 800 (t - 1)), j = 0..24 (the
// warp reads 64 consecutive samples per j). For the first frame of a clip, samples before the
// clip come from the carried tail (tail points one past its last sample) or are zero. Windowed
// as in step_a_load.
__device__ inline void step_a_load_global(int l, const float *base, const float *tail, int64_t start,
                                          const Tables &T, double (&ar)[25], double (&ai)[25]) {
  if (start >= 0) {
    // 8-byte loads from the 8-byte boundary at or below the frame start: when the frame starts
    // 4 bytes past one (mis = 1), lane l's pair is the high half of its own load and the low half
    // of lane l + 1's (lane 31: of lane 0's next load; the frame's last sample on its own); one
    // code path for either alignment
    const float *p0 = base + start;
    const uint32_t mis = (uint32_t)(reinterpret_cast<uintptr_t>(p0) >> 2) & 1u;
    const float2 *q = reinterpret_cast<const float2 *>(p0 - mis) + l;
    float2 v[25];
#pragma unroll
    for (int j = 0; j < 25; ++j) v[j] = __ldg(q + 32 * j);
    const float last = (mis && l == 31) ? __ldg(p0 + 1599) : 0.0f;
#pragma unroll
    for (int j = 0; j < 25; ++j) {
      const float nx = __shfl_sync(0xffffffffu, v[j].x, (l + 1) & 31);
      const float wx = __shfl_sync(0xffffffffu, j + 1 < 25 ? v[j + 1].x : last, 0);
      const float x0 = mis ? v[j].y : v[j].x;
      const float x1 = mis ? (l == 31 ? (j + 1 < 25 ? wx : last) : nx) : v[j].y;
      const double2 w = T.hann2[32 * j + l];  // periodic Hann at 64 j + 2 l and the next sample
      ar[j] = w.x * (double)x0;
      ai[j] = w.y * (double)x1;
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < 25; ++j) {
    const int n = 64 * j + 2 * l;  // even: n and n + 1 fall on the same side of sample 800
    float x0, x1;
    if (n >= 800) {  // first frame of a clip (start = -800): the new samples
      x0 = __ldg(base + (n - 800));
      x1 = __ldg(base + (n - 799));
    } else {  // ... after the carried tail or zeros
      x0 = tail ? __ldg(tail + (n - 800)) : 0.0f;
      x1 = tail ? __ldg(tail + (n - 799)) : 0.0f;
    }
    const double2 w = T.hann2[32 * j + l];  // periodic Hann at n and n + 1
    ar[j] = w.x * (double)x0;
    ai[j] = w.y * (double)x1;
  }
}

// Step A, first half for lane l: windowed z_{32 j + l} = (w s)[64 j + 2 l] + i (w s)[64 j + 2 l + 1]
// for j = 0..24 from the staged samples S (read before the buffer is overwritten).
__host__ __device__ inline void step_a_load(int l, const float *S, const Tables &T, double (&ar)[25],
                                            double (&ai)[25]) {
#pragma unroll
  for (int j = 0; j < 25; ++j) {
    const float2 x = *reinterpret_cast<const float2 *>(S + 64 * j + 2 * l);
    const double2 w = T.hann2[32 * j + l];  // periodic Hann at 64 j + 2 l and the next sample
    ar[j] = w.x * (double)x.x;
    ai[j] = w.y * (double)x.y;
  }
}

// Step A, second half: 25-point DFT over j, twiddle W_800^{l k1}, store to row k1, column l.
__host__ __device__ inline void step_a_dft(int l, const Tables &T, double (&ar)[25], double (&ai)[25], double2 *B) {
  // 25 = 5 x 5, j = j1 + 5 j2: inner DFTs over j2, result for (j1, ka) stored at j1 + 5 ka
#pragma unroll
  for (int j1 = 0; j1 < 5; ++j1)
    dft5(ar[j1], ai[j1], ar[j1 + 5], ai[j1 + 5], ar[j1 + 10], ai[j1 + 10], ar[j1 + 15], ai[j1 + 15], ar[j1 + 20],
         ai[j1 + 20]);
  // twiddle W_25^{j1 ka} = W_1600^{64 j1 ka}
#pragma unroll
  for (int j1 = 1; j1 < 5; ++j1)
#pragma unroll
    for (int ka = 1; ka < 5; ++ka) {
      const double2 w = tw(T, 64 * j1 * ka);
      cmul(ar[j1 + 5 * ka], ai[j1 + 5 * ka], w.x, w.y);
    }
  // outer DFTs over j1 for each ka (inputs at 5 ka + j1), output k1 = ka + 5 kb
#pragma unroll
  for (int ka = 0; ka < 5; ++ka) {
    double r[5], i[5];
#pragma unroll
    for (int j1 = 0; j1 < 5; ++j1) {
      r[j1] = ar[j1 + 5 * ka];
      i[j1] = ai[j1 + 5 * ka];
    }
    dft5(r[0], i[0], r[1], i[1], r[2], i[2], r[3], i[3], r[4], i[4]);
#pragma unroll
    for (int kb = 0; kb < 5; ++kb) {
      const int k1 = ka + 5 * kb;
      double yr = r[kb], yi = i[kb];
      if (k1 != 0) {
        const double2 w = T.twa[k1 * 32 + l];  // W_800^{l k1}
        cmul(yr, yi, w.x, w.y);
      }
      B[slot(k1, l)] = make_double2(yr, yi);
    }
  }
}

// Step C1, unit u = 4 k1 + l0 (0..99): 8-point DFT over l1 of row k1, columns l0 + 4 l1, times
// W_32^{l0 k2a}, written back to the same columns (output k2a in column l0 + 4 k2a). Units own
// disjoint columns, so a lane loads several units before storing any (the loads overlap).
__host__ __device__ inline void c1_load(int u, const double2 *B, double (&r)[8], double (&i)[8]) {
  const int k1 = u >> 2, l0 = u & 3;
#pragma unroll
  for (int l1 = 0; l1 < 8; ++l1) {
    const double2 v = B[slot(k1, l0 + 4 * l1)];
    r[l1] = v.x;
    i[l1] = v.y;
  }
}

__host__ __device__ inline void c1_finish(int u, const double2 (&w)[8], double (&r)[8], double (&i)[8], double2 *B) {
  const int k1 = u >> 2, l0 = u & 3;
  dft8(r, i);
#pragma unroll
  for (int k2a = 0; k2a < 8; ++k2a) {
    double xr = r[k2a], xi = i[k2a];
    if (l0 * k2a != 0) cmul(xr, xi, w[k2a].x, w[k2a].y);  // W_32^{l0 k2a}
    B[slot(k1, l0 + 4 * k2a)] = make_double2(xr, xi);
  }
}

// All C1 units of lane l: u = l, l + 32, l + 64 (loaded together), then l + 96 for l < 4. Every
// unit of the lane has l0 = l & 3, so its seven twiddles W_32^{l0 k2a} are read once.
__host__ __device__ inline void step_c1_lane(int l, const Tables &T, double2 *B) {
  double2 w[8];
#pragma unroll
  for (int k2a = 0; k2a < 8; ++k2a) w[k2a] = tw(T, 50 * (l & 3) * k2a);
  {
    double r[3][8], i[3][8];
#pragma unroll
    for (int q = 0; q < 3; ++q) c1_load(l + 32 * q, B, r[q], i[q]);
#pragma unroll
    for (int q = 0; q < 3; ++q) c1_finish(l + 32 * q, w, r[q], i[q], B);
  }
  if (l < 4) {
    double r[8], i[8];
    c1_load(l + 96, B, r, i);
    c1_finish(l + 96, w, r, i, B);
  }
}

// Step C2, unit u = 8 k1 + k2a (0..199): 4-point DFT over l0 of row k1, columns l0 + 4 k2a;
// output k2b goes to column k2b + 4 k2a. A lane loads all its (up to 7) units first.
__host__ __device__ inline void step_c2_lane(int l, double2 *B) {
  double2 x[7][4];
#pragma unroll
  for (int q = 0; q < 7; ++q) {
    const int u = l + 32 * q;
    if (u < 200) {
      const int k1 = u >> 3, k2a = u & 7;
#pragma unroll
      for (int l0 = 0; l0 < 4; ++l0) x[q][l0] = B[slot(k1, l0 + 4 * k2a)];
    }
  }
#pragma unroll
  for (int q = 0; q < 7; ++q) {
    const int u = l + 32 * q;
    if (u < 200) {
      const int k1 = u >> 3, k2a = u & 7;
      // X_k2b = sum_l0 x_l0 W_4^{l0 k2b}, W_4 = -i
      const double s02r = x[q][0].x + x[q][2].x, s02i = x[q][0].y + x[q][2].y;
      const double d02r = x[q][0].x - x[q][2].x, d02i = x[q][0].y - x[q][2].y;
      const double s13r = x[q][1].x + x[q][3].x, s13i = x[q][1].y + x[q][3].y;
      const double d13r = x[q][1].x - x[q][3].x, d13i = x[q][1].y - x[q][3].y;
      B[slot(k1, 0 + 4 * k2a)] = make_double2(s02r + s13r, s02i + s13i);
      B[slot(k1, 1 + 4 * k2a)] = make_double2(d02r + d13i, d02i - d13r);  // d02 - i d13
      B[slot(k1, 2 + 4 * k2a)] = make_double2(s02r - s13r, s02i - s13i);
      B[slot(k1, 3 + 4 * k2a)] = make_double2(d02r - d13i, d02i + d13r);  // d02 + i d13
    }
  }
}

// Step D for lane l: pairs (k, 800 - k). Round r = 1..12 takes Z at row r, column l
// (k = r + 25 k2 with k2 = (l >> 2) + 8 (l & 3)) and its partner Z_{800-k} at row 25 - r,
// column 31 - l; round 0 takes row 0 (k = 25 k2, k2 <= 16; the partner is Z_{800-k} in row 0).
// Rounds 0 and 1 are loaded first by every lane (rows 0, 1 and 24), so after a __syncwarp rows 0
// and 1 can hold the channel partials while rounds 2..12 are read one at a time.
struct Pair01 {
  double2 a0, b0, a1, b1;
};

__host__ __device__ inline int dk2(int l) { return (l >> 2) + 8 * (l & 3); }

__host__ __device__ inline void step_d_load01(int l, const double2 *B, Pair01 &R) {
  const int k2 = dk2(l);
  if (k2 <= 16) {
    R.a0 = B[slot(0, l)];
    R.b0 = B[zslot((800 - 25 * k2) % 800)];
  }
  R.a1 = B[slot(1, l)];
  R.b1 = B[slot(24, 31 - l)];
}


// |X_k|^2 of the real 1600-point DFT from a = Z_k and b = Z_{800-k}, with w = W_1600^k.
__host__ __device__ inline double power_bin(double2 w, double2 a, double2 b) {
  const double er = 0.5 * (a.x + b.x), ei = 0.5 * (a.y - b.y);  // (Z_k + conj Z_{800-k}) / 2
  const double dr = a.x - b.x, di = a.y + b.y;                    // Z_k - conj Z_{800-k}
  const double or_ = 0.5 * di, oi = -0.5 * dr;                    // / (2 i)
  const double xr = er + (or_ * w.x - oi * w.y);
  const double xi = ei + (or_ * w.y + oi * w.x);
  return xr * xr + xi * xi;
}

// Bin of lane l's run q at round r (-1 when the round has none): run 0 ascends from 25 k2, run 1
// descends from 800 - 25 k2; round 0 exists for k2 <= 16 (run 0) and k2 <= 15 (run 1: for
// k2 = 16 both would be bin 400).
__host__ __device__ inline int run_bin(int l, int q, int r) {
  const int k2 = dk2(l);
  if (r == 0 && (q == 0 ? k2 > 16 : k2 > 15)) return -1;
  return q == 0 ? 25 * k2 + r : 800 - 25 * k2 - r;
}

// Steps D and E for lane l: P of the lane's 26 bins (fp64 -> fp32) folded into channel partials.
// Each run carries two accumulators, for its current lower channel and the channel above; where
// the run enters a new channel (flush bit r) the finished one is written to its slot (ascending
// run: the lower; descending run: the upper); at the end of the run both are written.
__host__ __device__ inline void step_de_lane(int l, const Tables &T, const Pair01 &R, const double2 *B,
                                             float *part) {
  const int k2 = dk2(l);
  float lo[2] = {0.0f, 0.0f}, hi[2] = {0.0f, 0.0f};
  int nf[2] = {0, 0};
  const unsigned int fl[2] = {T.flush[l], T.flush[32 + l]};
  const unsigned short *sl[2] = {T.slot + (l * 2) * kMaxFlush, T.slot + (l * 2 + 1) * kMaxFlush};
#pragma unroll
  for (int r = 0; r < kRunLen; ++r) {
    const double2 a = r == 0 ? R.a0 : r == 1 ? R.a1 : B[slot(r, l)];
    const double2 b = r == 0 ? R.b0 : r == 1 ? R.b1 : B[slot(25 - r, 31 - l)];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      if (r == 0 && (q == 0 ? k2 > 16 : k2 > 15)) continue;
      const double2 w = T.twd[(q * kRunLen + r) * 32 + l];  // W_1600^k (run 0), W_1600^{800-k} (run 1)
      const float p = q == 0 ? (float)power_bin(w, a, b) : (float)power_bin(w, b, a);
      if ((fl[q] >> r) & 1u) {
        if (q == 0) {
          part[sl[0][nf[0]++]] = lo[0];
          lo[0] = hi[0];
          hi[0] = 0.0f;
        } else {
          part[sl[1][nf[1]++]] = hi[1];
          hi[1] = lo[1];
          lo[1] = 0.0f;
        }
      }
      const float2 mw = T.melw2[(q * kRunLen + r) * 32 + l];
      lo[q] = fmaf(mw.x, p, lo[q]);
      hi[q] = fmaf(mw.y, p, hi[q]);
    }
  }
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    part[sl[q][nf[q]++]] = lo[q];
    part[sl[q][nf[q]]] = hi[q];
  }
}

// Step E, second half: channel b = lane, lane + 32, lane + 64 adds its partials, then log10,
// clamp and quantise.
// Level of a clamped log-mel value: mode 0 floor((L - lmin) * 16 / range) (for the default
// [-7, 2] the same fp32 operations as (L + 7) * 16 / 9), mode 1 the nearest of 16 reconstruction
// points lmin + k range / 15 (ties upward), mode 2 mu-law companding of u = (L - lmin) / range
// followed by 16 uniform levels.
__host__ __device__ inline int quant_level(float L, const Quant &q) {
  float y;
  if (q.mode == 1) {
    y = (L - q.lmin) * 15.0f / q.range + 0.5f;
  } else if (q.mode == 2) {
    y = 16.0f * (log1pf(q.mu * ((L - q.lmin) / q.range)) * q.inv_log1p_mu);
  } else {
    y = (L - q.lmin) * 16.0f / q.range;
  }
  const int c = (int)floorf(y);
  return c > 15 ? 15 : (c < 0 ? 0 : c);
}

__host__ __device__ inline void step_e_codes(int l, const Tables &T, const float *part, uint8_t *codes_row,
                                             double *lhat_row, const Quant &qz) {
  for (int b = l; b < kMel; b += 32) {
    float m = 0.0f;
    for (int q = T.chanseg[b]; q < T.chanseg[b + 1]; ++q) m += part[q];
    float L = log10f(fmaxf(m, 1e-10f));  // fmaxf drops a NaN energy
    L = fminf(fmaxf(L, qz.lmin), qz.lmax);
    const int c = quant_level(L, qz);
    codes_row[b] = (uint8_t)c;
    if (lhat_row) lhat_row[b] = (double)L;
  }
}

// ---------------------------------------------------------------- host tables

struct HostTables {
  std::vector<double2> w, hann2, twa;
  std::vector<float2> melw2;
  std::vector<double2> twd;
  std::vector<unsigned short> slot;
  std::vector<unsigned int> flush;
  int chanseg[81];
  bool ok = true;  // every check of the mel layout held
  Tables view() const {
    return Tables{w.data(), hann2.data(), twa.data(), melw2.data(), twd.data(), slot.data(), flush.data(), chanseg};
  }
};

void build_host_tables(HostTables &H) {
  const double two_pi = 6.283185307179586476925286766559;
  H.w.resize(kBins);
  for (int k = 0; k < kBins; ++k) H.w[k] = make_double2(std::cos(two_pi * k / 1600), -std::sin(two_pi * k / 1600));
  H.hann2.resize(800);
  for (int m = 0; m < 800; ++m)
    H.hann2[m] = make_double2(0.5 - 0.5 * std::cos(two_pi * (2 * m) / 1600), 0.5 - 0.5 * std::cos(two_pi * (2 * m + 1) / 1600));
  H.twa.resize(800);
  for (int k1 = 0; k1 < 25; ++k1)
    for (int l = 0; l < 32; ++l) {
      const int j = (l * k1) % 800;
      H.twa[k1 * 32 + l] = make_double2(std::cos(two_pi * j / 800), -std::sin(two_pi * j / 800));
    }
  // HTK mel points: 82 points equally spaced in mel on [0, 8000] Hz; triangle b rises from point
  // b to its peak (1) at point b + 1 and falls to point b + 2, evaluated at f_k = 10 k Hz
  const double mel_top = 2595.0 * std::log10(1.0 + 8000.0 / 700.0);
  double fp[kMel + 2];
  for (int i = 0; i < kMel + 2; ++i) fp[i] = 700.0 * (std::pow(10.0, (mel_top * i / (kMel + 1)) / 2595.0) - 1.0);
  auto tri = [&](int b, int k) {  // weight of bin k in channel b (0 outside the triangle)
    if (b < 0 || b >= kMel) return 0.0;
    const double f = 10.0 * k;
    const double up = (f - fp[b]) / (fp[b + 1] - fp[b]);
    const double down = (fp[b + 2] - f) / (fp[b + 2] - fp[b + 1]);
    const double h = up < down ? up : down;
    return h > 0.0 ? h : 0.0;
  };
  // every bin k lies in one gap (fp[g], fp[g + 1]] (g = -1 for bin 0): it can feed channel g - 1
  // (falling edge) and channel g (rising edge) only; lower channel of bin k: g - 1
  std::vector<int> chl(kBins);
  for (int k = 0; k < kBins; ++k) {
    int g = -1;
    while (g + 1 < kMel + 1 && fp[g + 1] < 10.0 * k) ++g;
    chl[k] = g - 1;
    for (int b = 0; b < kMel; ++b)  // no weight outside the two channels of the gap
      if (b != g - 1 && b != g && tri(b, k) != 0.0) H.ok = false;
  }
  // per lane and run: weights, the rounds where the run enters a new channel, the channel of each
  // partial it writes (-1 / 80: outside 0..79, sent to a trash slot)
  H.melw2.assign(2 * kRunLen * 32, make_float2(0.0f, 0.0f));
  H.twd.assign(2 * kRunLen * 32, make_double2(0.0, 0.0));
  for (int l = 0; l < 32; ++l)
    for (int q = 0; q < 2; ++q)
      for (int r = 0; r < kRunLen; ++r) {
        const int k = run_bin(l, q, r);  // at most 800: a direct entry of the W table
        if (k >= 0) H.twd[(q * kRunLen + r) * 32 + l] = H.w[k];
      }
  H.flush.assign(64, 0u);
  std::vector<int> fch[32][2];
  for (int l = 0; l < 32; ++l)
    for (int q = 0; q < 2; ++q) {
      int prev = -100, c = 0;
      for (int r = 0; r < kRunLen; ++r) {
        const int k = run_bin(l, q, r);
        if (k < 0) continue;
        c = chl[k];
        H.melw2[(q * kRunLen + r) * 32 + l] = make_float2((float)tri(c, k), (float)tri(c + 1, k));
        if (prev != -100 && c != prev) {
          if (c != prev + (q == 0 ? 1 : -1)) H.ok = false;  // one channel per step
          H.flush[q * 32 + l] |= 1u << r;
          fch[l][q].push_back(q == 0 ? prev : prev + 1);  // the channel that is finished
        }
        prev = c;
      }
      fch[l][q].push_back(c);
      fch[l][q].push_back(c + 1);
      if ((int)fch[l][q].size() > kMaxFlush) H.ok = false;
    }
  // slots numbered channel by channel (lane, run and order within the run ascending), so that
  // channel b adds the contiguous slots [chanseg[b], chanseg[b + 1]); then one trash slot
  H.slot.assign(32 * 2 * kMaxFlush, 0);
  int nslot = 0;
  for (int b = 0; b < kMel; ++b) {
    H.chanseg[b] = nslot;
    for (int l = 0; l < 32; ++l)
      for (int q = 0; q < 2; ++q)
        for (size_t i = 0; i < fch[l][q].size(); ++i)
          if (fch[l][q][i] == b) H.slot[(l * 2 + q) * kMaxFlush + i] = (unsigned short)nslot++;
  }
  H.chanseg[kMel] = nslot;
  for (int l = 0; l < 32; ++l)
    for (int q = 0; q < 2; ++q)
      for (size_t i = 0; i < fch[l][q].size(); ++i)
        if (fch[l][q][i] < 0 || fch[l][q][i] >= kMel) H.slot[(l * 2 + q) * kMaxFlush + i] = (unsigned short)nslot;
  if (nslot + 1 > kMaxSegs) H.ok = false;
}

const HostTables &host_tables() {
  static HostTables H;
  static std::once_flag once;
  std::call_once(once, [] { build_host_tables(H); });
  return H;
}

std::mutex g_upload_mu;
bool g_uploaded[256] = {false};

cudaError_t ensure_device_tables() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_upload_mu);
  if (g_uploaded[dev]) return cudaSuccess;
  const HostTables &H = host_tables();
  if (!H.ok) return cudaErrorInvalidValue;
  if ((e = cudaMemcpyToSymbol(d_w1600, H.w.data(), sizeof(double2) * kBins)) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_hann2, H.hann2.data(), sizeof(double2) * 800)) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_twa, H.twa.data(), sizeof(double2) * 800)) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_melw2, H.melw2.data(), sizeof(float2) * H.melw2.size())) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_twd, H.twd.data(), sizeof(double2) * H.twd.size())) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_slot, H.slot.data(), sizeof(unsigned short) * H.slot.size())) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_flush, H.flush.data(), sizeof(unsigned int) * H.flush.size())) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_chanseg, H.chanseg, sizeof(H.chanseg))) != cudaSuccess) return e;
  g_uploaded[dev] = true;
  return cudaSuccess;
}

// Carried tail of clip c into tails_out row c, by threads tid = 0..NT-1 of a warp or block: the
// last 800 consumed samples of the clip (those ending at sample 800 F), the tail in when the clip
// has no frame, zeros when there is neither; zeros and an offsets error when the clip is shorter
// than its frames need. The aligned copy issues all of a thread's loads before its stores.
template <int NT>
__device__ void clip_tail(int c, const float *__restrict__ wav, const int64_t *__restrict__ soff,
                          const int64_t *__restrict__ foff, const float *tails, float *tails_out, uint32_t *err,
                          int tid) {
  constexpr int nt = NT, PER = (kHop / 4 + NT - 1) / NT;
  const int64_t F = foff[c + 1] - foff[c];
  const int64_t len = soff[c + 1] - soff[c];
  float *dst = tails_out + (int64_t)c * kHop;
  if (F >= 1 && (int64_t)kHop * F > len) {
    if (tid == 0) record_error(err, DMEL_DEVERR_OFFSETS);
    for (int n = tid; n < kHop; n += nt) dst[n] = 0.0f;
    return;
  }
  const float *src = F >= 1 ? wav + soff[c] + (int64_t)kHop * (F - 1) : (tails ? tails + (int64_t)c * kHop : nullptr);
  if (!src) {
    for (int n = tid; n < kHop; n += nt) dst[n] = 0.0f;
  } else if ((reinterpret_cast<uintptr_t>(src) & 15) == 0 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
    float4 v[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k)
      if (tid + k * NT < kHop / 4) v[k] = reinterpret_cast<const float4 *>(src)[tid + k * NT];
#pragma unroll
    for (int k = 0; k < PER; ++k)
      if (tid + k * NT < kHop / 4) reinterpret_cast<float4 *>(dst)[tid + k * NT] = v[k];
  } else {
    for (int n = tid; n < kHop; n += nt) dst[n] = src[n];
  }
}

}  // namespace

// ---------------------------------------------------------------- kernels

template <int kWarpsPerBlock>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, 1) codes_kernel_entry(const float *__restrict__ wav,
                                                                             const int64_t *__restrict__ soff,
                                                                             const int64_t *__restrict__ foff,
                                                                             int n_clips, int64_t n_frames,
                                                                             const float *__restrict__ tails,
                                                                             float *__restrict__ tails_out,
                                                                             uint8_t *__restrict__ codes,
                                                                             Quant qz, uint32_t *err) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // constant tables: global -> shared once per block
  {
    double2 *w = reinterpret_cast<double2 *>(smem + kSmW);
    double2 *h2 = reinterpret_cast<double2 *>(smem + kSmHann);
    double2 *ta = reinterpret_cast<double2 *>(smem + kSmTwA);
    float2 *mw = reinterpret_cast<float2 *>(smem + kSmMelW2);
    unsigned short *sl = reinterpret_cast<unsigned short *>(smem + kSmSlot);
    unsigned int *fl = reinterpret_cast<unsigned int *>(smem + kSmFlush);
    int *cs = reinterpret_cast<int *>(smem + kSmChanSeg);
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) w[i] = d_w1600[i];
    for (int i = threadIdx.x; i < 800; i += blockDim.x) {
      h2[i] = d_hann2[i];
      ta[i] = d_twa[i];
    }
    double2 *td = reinterpret_cast<double2 *>(smem + kSmTwD);
    for (int i = threadIdx.x; i < 2 * kRunLen * 32; i += blockDim.x) {
      mw[i] = d_melw2[i];
      td[i] = d_twd[i];
    }
    for (int i = threadIdx.x; i < 32 * 2 * kMaxFlush; i += blockDim.x) sl[i] = d_slot[i];
    for (int i = threadIdx.x; i < 64; i += blockDim.x) fl[i] = d_flush[i];
    for (int i = threadIdx.x; i < 81; i += blockDim.x) cs[i] = d_chanseg[i];
  }
  __syncthreads();
  const Tables T{reinterpret_cast<const double2 *>(smem + kSmW), reinterpret_cast<const double2 *>(smem + kSmHann),
                 reinterpret_cast<const double2 *>(smem + kSmTwA), reinterpret_cast<const float2 *>(smem + kSmMelW2),
                 reinterpret_cast<const double2 *>(smem + kSmTwD),
                 reinterpret_cast<const unsigned short *>(smem + kSmSlot),
                 reinterpret_cast<const unsigned int *>(smem + kSmFlush), reinterpret_cast<const int *>(smem + kSmChanSeg)};
  double2 *B = reinterpret_cast<double2 *>(smem + kSmTables + warp * kWarpBufBytes);
  float *part = reinterpret_cast<float *>(B);  // channel partials: rows 0 and 1, once rounds 0 and 1 are read

  const int64_t warps_total = (int64_t)gridDim.x * kWarpsPerBlock;
  const int64_t gw = (int64_t)blockIdx.x * kWarpsPerBlock + warp;
  const int64_t chunk = (n_frames + warps_total - 1) / warps_total;
  // tails_out (never the tails in): written after the frames, by the warps that have no frame
  // when there are enough of them (a tail copy costs a fraction of a frame: at most 4 chunk clips
  // each), else by every warp, clip c by warp c mod warps_total
  auto tails_after = [&]() {
    if (!tails_out) return;
    const int64_t busy = (n_frames + chunk - 1) / chunk, idle = warps_total - busy;
    const bool by_idle = idle > 0 && (n_clips + idle - 1) / idle <= 4 * chunk;
    const int64_t w = by_idle ? gw - busy : gw, nw = by_idle ? idle : warps_total;
    if (w < 0) return;
    for (int64_t c = w; c < n_clips; c += nw) clip_tail<32>((int)c, wav, soff, foff, tails, tails_out, err, lane);
  };
  const int64_t g0 = gw * chunk;
  const int64_t g1 = g0 + chunk < n_frames ? g0 + chunk : n_frames;
  if (g0 >= g1) {
    tails_after();
    return;
  }

  // last clip with foff[clip] <= g0: a 32-way search, each lane probing one point per round
  int lo = 0, hi = n_clips - 1;
  while (hi - lo > 31) {
    const int64_t span = hi - lo;
    const int probe = lo + (int)((span * (lane + 1)) / 33);
    const unsigned le = __ballot_sync(0xffffffffu, foff[probe] <= g0);
    if (le == 0) {
      hi = lo + (int)((span * 1) / 33) - 1;
    } else {
      const int top = 31 - __clz(le);  // last probe with foff <= g0 (foff is non-decreasing)
      const int nlo = lo + (int)((span * (top + 1)) / 33);
      const int nhi = top == 31 ? hi : lo + (int)((span * (top + 2)) / 33) - 1;
      lo = nlo;
      hi = nhi;
    }
  }
  {
    const int probe = lo + lane;
    const unsigned le = __ballot_sync(0xffffffffu, probe <= hi && foff[probe] <= g0);
    lo = lo + (31 - __clz(le));
  }
  int clip = lo;
  // the clip's bounds stay in registers while the warp walks its frames (four independent loads
  // when it enters a clip, none per frame)
  int64_t f_next, f_first, s_first, s_len;
  auto enter = [&]() {
    f_next = clip + 1 < n_clips ? foff[clip + 1] : INT64_MAX;
    f_first = foff[clip];
    s_first = soff[clip];
    s_len = soff[clip + 1] - s_first;
  };
  enter();

  for (int64_t g = g0; g < g1; ++g) {
    if (g >= f_next) {  // the next clip with a frame at or before g (clips of no frame skipped)
      do ++clip; while (clip + 1 < n_clips && foff[clip + 1] <= g);
      enter();
    }
    const int64_t t = g - f_first;
    const int64_t len = s_len;
    uint8_t *crow = codes + g * kMel;
    if (t < 0 || (int64_t)kHop * (t + 1) > len) {  // offsets do not describe this frame
      if (lane == 0) record_error(err, DMEL_DEVERR_OFFSETS);
      for (int b = lane; b < kMel; b += 32) crow[b] = 0;
      continue;
    }
    // the next frame of this clip needs samples [800 (t + 1), 800 (t + 2)): start them into L1
    if (g + 1 < g1 && (int64_t)kHop * (t + 2) <= len && lane < 25)
      asm volatile("prefetch.global.L1 [%0];" ::"l"(wav + s_first + (int64_t)kHop * (t + 1) + 32 * lane));
    __syncwarp();  // the previous frame's partials are read before this frame's DFT outputs land
    {
      double ar[25], ai[25];
      step_a_load_global(lane, wav + s_first, tails ? tails + (int64_t)clip * kHop + kHop : nullptr,
                         (int64_t)kHop * (t - 1), T, ar, ai);
      step_a_dft(lane, T, ar, ai, B);
    }
    __syncwarp();
    step_c1_lane(lane, T, B);
    __syncwarp();
    step_c2_lane(lane, B);
    __syncwarp();
    {
      Pair01 R;
      step_d_load01(lane, B, R);
      __syncwarp();  // rows 0, 1 and 24 are read before the partials overwrite rows 0 and 1
      step_de_lane(lane, T, R, B, part);
    }
    __syncwarp();
    step_e_codes(lane, T, part, crow, nullptr, qz);
    __syncwarp();
  }
  tails_after();
}

// Carried tails: one block per clip row (800 floats); the source is the last 800 consumed
// samples of the clip, or the tail in when the clip has no frame.
__global__ void __launch_bounds__(256) tails_kernel_entry(const float *__restrict__ wav,
                                                          const int64_t *__restrict__ soff,
                                                          const int64_t *__restrict__ foff, int n_clips,
                                                          const float *tails, float *tails_out, uint32_t *err) {
  for (int c = blockIdx.x; c < n_clips; c += gridDim.x)
    clip_tail<256>(c, wav, soff, foff, tails, tails_out, err, threadIdx.x);
}

// ---------------------------------------------------------------- host entry points

cudaError_t launch_codes(const float *wav, const int64_t *soff, const int64_t *foff, int n_clips, int64_t n_frames,
                         const float *tails, float *tails_out, uint8_t *codes, uint32_t *err, int num_sms,
                         cudaStream_t stream, int *launches, Quant q) {
  cudaError_t e = ensure_device_tables();
  if (e != cudaSuccess) return e;
  static std::atomic<bool> attr[256];
  if ((e = set_smem_attr_once(codes_kernel_entry<kWarpsDefault>, smem_bytes(kWarpsDefault), attr)) != cudaSuccess)
    return e;
  // the codes kernel writes the carried tails itself (after its frames) unless tails_out overlaps
  // the tails in, whose rows other warps may still have to read: then a kernel of its own after it
  const uintptr_t ti = reinterpret_cast<uintptr_t>(tails), to = reinterpret_cast<uintptr_t>(tails_out);
  const uintptr_t tb = (uintptr_t)n_clips * kHop * sizeof(float);
  const bool overlap = tails && tails_out && ti < to + tb && to < ti + tb;
  const bool fused = tails_out && n_clips > 0 && n_frames > 0 && !overlap;
  if (n_frames > 0) {
    int64_t blocks = (n_frames + kWarpsDefault - 1) / kWarpsDefault;
    if (blocks > num_sms) blocks = num_sms;  // one persistent block per SM
    codes_kernel_entry<kWarpsDefault><<<(unsigned)blocks, kWarpsDefault * 32, smem_bytes(kWarpsDefault), stream>>>(
        wav, soff, foff, n_clips, n_frames, tails, fused ? tails_out : nullptr, codes, q, err);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ++*launches;
  }
  if (tails_out && n_clips > 0 && !fused) {
    int64_t blocks = n_clips;
    if (blocks > (int64_t)num_sms * 16) blocks = (int64_t)num_sms * 16;
    tails_kernel_entry<<<(unsigned)blocks, 256, 0, stream>>>(wav, soff, foff, n_clips, tails, tails_out, err);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ++*launches;
  }
  return cudaSuccess;
}

// Host emulation of the per-frame arithmetic of codes_kernel_entry (the same step functions;
// the lanes and units of each step run one after another, and a step's loads all complete
// before its stores where the kernel separates them with __syncwarp). Diagnostic only: no
// entry point of the front end calls it.
void emulate_codes_frame_host(const float *frame1600, uint8_t *codes80, double *lhat80, Quant q) {
  const HostTables &H = host_tables();
  const Tables T = H.view();
  std::vector<double2> B(800);
  std::vector<Pair01> R(32);
  std::vector<float> part(kMaxSegs, 0.0f);
  std::vector<double> arb(32 * 25), aib(32 * 25);
  for (int l = 0; l < 32; ++l)
    step_a_load(l, frame1600, T, *reinterpret_cast<double(*)[25]>(&arb[25 * l]),
                *reinterpret_cast<double(*)[25]>(&aib[25 * l]));
  for (int l = 0; l < 32; ++l)
    step_a_dft(l, T, *reinterpret_cast<double(*)[25]>(&arb[25 * l]), *reinterpret_cast<double(*)[25]>(&aib[25 * l]),
               B.data());
  for (int l = 0; l < 32; ++l) step_c1_lane(l, T, B.data());
  for (int l = 0; l < 32; ++l) step_c2_lane(l, B.data());
  for (int l = 0; l < 32; ++l) step_d_load01(l, B.data(), R[l]);
  for (int l = 0; l < 32; ++l) step_de_lane(l, T, R[l], B.data(), reinterpret_cast<float *>(B.data()));
  for (int i = 0; i < kMaxSegs; ++i) part[i] = reinterpret_cast<const float *>(B.data())[i];
  for (int l = 0; l < 32; ++l) step_e_codes(l, T, part.data(), codes80, lhat80, q);
}

}  // namespace dmel
