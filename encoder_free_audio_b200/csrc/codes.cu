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
//       Z_{800-k} at row 25 - r, column 31 - l (both bank-conflict free);
//   E   the 1571 non-zero mel weights, as one list sorted by channel, are cut into 32 equal
//       chunks; lane l sums its chunk into per-channel partials, then 80 channel sums, log10,
//       clamp, quantise (fp32).
// Each frame's 1600 samples are first copied into the warp's buffer with coalesced loads.
// Every root of unity comes from one fp64 table of W_1600^k, k = 0..800 (W_800 = W_1600^2,
// W_32 = W_1600^50, W_25 = W_1600^64, W^{1600 - k} = conj W^k). The buffer is swizzled so the
// column accesses of A, C1 and C2 are free of shared-memory bank conflicts.
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace dmel {
namespace {

#ifndef DMEL_CODES_WARPS
#define DMEL_CODES_WARPS 12
#endif
constexpr int kWarpsPerBlock = DMEL_CODES_WARPS;
constexpr int kMelNnzMax = 1600;
constexpr int kMaxSegs = 128;      // channel segments of the 32 mel chunks (<= 80 + 31)

// Shared memory of one block: the constant tables once, then one 800-element complex buffer
// per warp (Y, then Z in place, then P in place; the mel partials follow P).
constexpr int kSmW = 0;                                    // double2 [801]: W_1600^k
constexpr int kSmHann = kSmW + 801 * 16;                   // double2 [800]: (w[2m], w[2m+1])
constexpr int kSmTwA = kSmHann + 800 * 16;                 // double2 [25 * 32]: W_800^{l k1}
constexpr int kSmMelW = kSmTwA + 800 * 16;                 // float [kMelNnzMax]: weights
constexpr int kSmMelK = kSmMelW + kMelNnzMax * 4;          // short [kMelNnzMax]: bin of each weight
constexpr int kSmMelB = kSmMelK + kMelNnzMax * 2;          // uchar [kMelNnzMax]: channel of each weight
constexpr int kSmChunk = kSmMelB + kMelNnzMax;             // int [33]: chunk bounds per lane
constexpr int kSmSegFirst = kSmChunk + 36 * 4;             // int [33]: first segment of each lane
constexpr int kSmChanSeg = kSmSegFirst + 36 * 4;           // int [81]: segment range per channel
constexpr int kSmTables = (kSmChanSeg + 84 * 4 + 127) / 128 * 128;
constexpr int kWarpBufBytes = 800 * 16;
constexpr int kPartOffset = 3216;                          // mel partials (floats) after P[801]
constexpr int kSmemBytes = kSmTables + kWarpsPerBlock * kWarpBufBytes;
static_assert(kPartOffset + kMaxSegs * 4 <= kWarpBufBytes, "mel partials fit behind P");
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

// Constant tables, filled once per device from host-computed fp64 values.
__device__ double2 d_w1600[kBins];
__device__ double2 d_hann2[800];
__device__ double2 d_twa[800];
__device__ float d_melw[kMelNnzMax];
__device__ short d_melk[kMelNnzMax];
__device__ unsigned char d_melb[kMelNnzMax];
__device__ int d_chunk[33];
__device__ int d_segfirst[33];
__device__ int d_chanseg[81];

struct Tables {
  const double2 *w;      // W_1600^k = exp(-2 pi i k / 1600), k = 0..800
  const double2 *hann2;  // periodic Hann pairs (w[2m], w[2m+1]), m = 0..799
  const double2 *twa;    // W_800^{l k1} at [k1 * 32 + l]
  const float *melw;     // non-zero mel weights (fp32), sorted by channel then bin
  const short *melk;     // their bins
  const unsigned char *melb;  // their channels
  const int *chunk;      // lane l sums entries [chunk[l], chunk[l + 1])
  const int *segfirst;   // lane l owns the partial-sum slots [segfirst[l], segfirst[l + 1])
  const int *chanseg;    // channel b adds the partials [chanseg[b], chanseg[b + 1])
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

// Copies the 1600 raw samples of frame t of a clip, x[800 (t - 1) + n], into S[n] with
// coalesced loads (lane l takes n = l + 32 i). Samples before the clip come from the carried
// tail (tail points one past its last sample) or are zero.
__device__ inline void stage_frame(int l, const float *base, const float *tail, int64_t start, float *S) {
  if (start >= 0) {
    const float *src = base + start;
#pragma unroll 10
    for (int n = l; n < 1600; n += 32) S[n] = __ldg(src + n);
  } else {
    // first frame of a clip (start = -800): the carried tail (or zeros), then the new samples
#pragma unroll 5
    for (int n = l; n < 800; n += 32) S[n] = tail ? __ldg(tail + (n - 800)) : 0.0f;
#pragma unroll 5
    for (int n = 800 + l; n < 1600; n += 32) S[n] = __ldg(base + (n - 800));
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
// disjoint columns, so a lane loads two units before storing either (the loads overlap).
__host__ __device__ inline void c1_load(int u, const double2 *B, double (&r)[8], double (&i)[8]) {
  const int k1 = u >> 2, l0 = u & 3;
#pragma unroll
  for (int l1 = 0; l1 < 8; ++l1) {
    const double2 v = B[slot(k1, l0 + 4 * l1)];
    r[l1] = v.x;
    i[l1] = v.y;
  }
}

__host__ __device__ inline void c1_finish(int u, const Tables &T, double (&r)[8], double (&i)[8], double2 *B) {
  const int k1 = u >> 2, l0 = u & 3;
  dft8(r, i);
#pragma unroll
  for (int k2a = 0; k2a < 8; ++k2a) {
    double xr = r[k2a], xi = i[k2a];
    if (l0 * k2a != 0) {
      const double2 w = tw(T, 50 * l0 * k2a);  // W_32^{l0 k2a}
      cmul(xr, xi, w.x, w.y);
    }
    B[slot(k1, l0 + 4 * k2a)] = make_double2(xr, xi);
  }
}

// All C1 units of lane l: u = l, l + 32, l + 64 (and l + 96 for l < 4), two at a time.
__host__ __device__ inline void step_c1_lane(int l, const Tables &T, double2 *B) {
#pragma unroll
  for (int q = 0; q < 4; q += 2) {
    const int u0 = l + 32 * q, u1 = l + 32 * (q + 1);
    double r0[8], i0[8], r1[8], i1[8];
    const bool has1 = u1 < 100;
    c1_load(u0, B, r0, i0);
    if (has1) c1_load(u1, B, r1, i1);
    c1_finish(u0, T, r0, i0, B);
    if (has1) c1_finish(u1, T, r1, i1, B);
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

// Step D, first half for lane l: pairs (k, 800 - k). Round r = 1..12 takes Z at row r, column
// l (k = r + 25 k2 with k2 = (l >> 2) + 8 (l & 3)) and its partner Z_{800-k} at row 25 - r,
// column 31 - l; round 0 takes row 0 (k = 25 k2, k2 <= 16; the partner is Z_{800-k} in row 0).
struct PairRegs {
  double2 a[13], b[13];
};

__host__ __device__ inline int dk2(int l) { return (l >> 2) + 8 * (l & 3); }

__host__ __device__ inline void step_d_load(int l, const double2 *B, PairRegs &R) {
  const int k2 = dk2(l);
  if (k2 <= 16) {
    R.a[0] = B[slot(0, l)];
    R.b[0] = B[zslot((800 - 25 * k2) % 800)];
  }
#pragma unroll
  for (int r = 1; r <= 12; ++r) {
    R.a[r] = B[slot(r, l)];
    R.b[r] = B[slot(25 - r, 31 - l)];
  }
}

// |X_k|^2 of the real 1600-point DFT from a = Z_k and b = Z_{800-k}.
__host__ __device__ inline double power_bin(const Tables &T, int k, double2 a, double2 b) {
  const double er = 0.5 * (a.x + b.x), ei = 0.5 * (a.y - b.y);  // (Z_k + conj Z_{800-k}) / 2
  const double dr = a.x - b.x, di = a.y + b.y;                    // Z_k - conj Z_{800-k}
  const double or_ = 0.5 * di, oi = -0.5 * dr;                    // / (2 i)
  const double2 w = tw(T, k);
  const double xr = er + (or_ * w.x - oi * w.y);
  const double xi = ei + (or_ * w.y + oi * w.x);
  return xr * xr + xi * xi;
}

// Step D, second half: P_k and P_{800 - k} (fp32) in natural order over the buffer.
__host__ __device__ inline void step_d_store(int l, const Tables &T, const PairRegs &R, float *P) {
  const int k2 = dk2(l);
  if (k2 <= 16) {
    const int k = 25 * k2;
    P[k] = (float)power_bin(T, k, R.a[0], R.b[0]);
    if (k != 400) P[800 - k] = (float)power_bin(T, 800 - k, R.b[0], R.a[0]);
  }
#pragma unroll
  for (int r = 1; r <= 12; ++r) {
    const int k = r + 25 * k2;
    P[k] = (float)power_bin(T, k, R.a[r], R.b[r]);
    P[800 - k] = (float)power_bin(T, 800 - k, R.b[r], R.a[r]);
  }
}

// Step E, first half for lane l: the entries [chunk[l], chunk[l + 1]) of the weight list,
// summed per channel into the partial-sum slots segfirst[l], segfirst[l] + 1, ... Every lane
// walks the same number of entries (within one), so the loop does not diverge.
__host__ __device__ inline void step_e_chunk(int l, const Tables &T, const float *P, float *part) {
  const int e0 = T.chunk[l], e1 = T.chunk[l + 1];
  int seg = T.segfirst[l];
  int cur = T.melb[e0];
  float acc = 0.0f;
#pragma unroll 4
  for (int e = e0; e < e1; ++e) {
    const float v = T.melw[e] * P[T.melk[e]];
    const int b = T.melb[e];
    if (b != cur) {
      part[seg++] = acc;
      acc = 0.0f;
      cur = b;
    }
    acc += v;
  }
  part[seg] = acc;
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
  std::vector<float> melw;
  std::vector<short> melk;
  std::vector<unsigned char> melb;
  int chunk[33], segfirst[33], chanseg[81];
  Tables view() const {
    return Tables{w.data(), hann2.data(), twa.data(), melw.data(), melk.data(), melb.data(), chunk, segfirst, chanseg};
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
  // HTK mel points: 82 points equally spaced in mel on [0, 8000] Hz; non-zero triangle weights
  // listed channel by channel, bins ascending
  const double mel_top = 2595.0 * std::log10(1.0 + 8000.0 / 700.0);
  double fp[kMel + 2];
  for (int i = 0; i < kMel + 2; ++i) fp[i] = 700.0 * (std::pow(10.0, (mel_top * i / (kMel + 1)) / 2595.0) - 1.0);
  H.melw.clear();
  H.melk.clear();
  H.melb.clear();
  for (int b = 0; b < kMel; ++b)
    for (int k = 0; k < kBins; ++k) {
      const double f = 10.0 * k;
      const double up = (f - fp[b]) / (fp[b + 1] - fp[b]);
      const double down = (fp[b + 2] - f) / (fp[b + 2] - fp[b + 1]);
      const double h = up < down ? up : down;
      if (h > 0.0) {
        H.melw.push_back((float)h);
        H.melk.push_back((short)k);
        H.melb.push_back((unsigned char)b);
      }
    }
  const int nnz = (int)H.melw.size();
  for (int l = 0; l <= 32; ++l) H.chunk[l] = (int)((int64_t)l * nnz / 32);
  // partial-sum slots: one per maximal run of one channel inside a chunk, numbered lane by lane
  int seg = 0;
  for (int b = 0; b <= kMel; ++b) H.chanseg[b] = -1;
  for (int l = 0; l < 32; ++l) {
    H.segfirst[l] = seg;
    for (int e = H.chunk[l]; e < H.chunk[l + 1]; ++e) {
      if (e > H.chunk[l] && H.melb[e] != H.melb[e - 1]) ++seg;
      if (H.chanseg[H.melb[e]] < 0) H.chanseg[H.melb[e]] = seg;
    }
    ++seg;
  }
  H.segfirst[32] = seg;
  H.chanseg[kMel] = seg;
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
  if (H.melw.size() > (size_t)kMelNnzMax || H.chanseg[kMel] > kMaxSegs) return cudaErrorInvalidValue;
  if ((e = cudaMemcpyToSymbol(d_w1600, H.w.data(), sizeof(double2) * kBins)) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_hann2, H.hann2.data(), sizeof(double2) * 800)) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_twa, H.twa.data(), sizeof(double2) * 800)) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_melw, H.melw.data(), sizeof(float) * H.melw.size())) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_melk, H.melk.data(), sizeof(short) * H.melk.size())) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_melb, H.melb.data(), H.melb.size())) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_chunk, H.chunk, sizeof(H.chunk))) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_segfirst, H.segfirst, sizeof(H.segfirst))) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_chanseg, H.chanseg, sizeof(H.chanseg))) != cudaSuccess) return e;
  g_uploaded[dev] = true;
  return cudaSuccess;
}

}  // namespace

// ---------------------------------------------------------------- kernels

__global__ void __launch_bounds__(kWarpsPerBlock * 32, 1) codes_kernel_entry(const float *__restrict__ wav,
                                                                             const int64_t *__restrict__ soff,
                                                                             const int64_t *__restrict__ foff,
                                                                             int n_clips, int64_t n_frames,
                                                                             const float *__restrict__ tails,
                                                                             uint8_t *__restrict__ codes,
                                                                             Quant qz, uint32_t *err) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // constant tables: global -> shared once per block
  {
    double2 *w = reinterpret_cast<double2 *>(smem + kSmW);
    double2 *h2 = reinterpret_cast<double2 *>(smem + kSmHann);
    double2 *ta = reinterpret_cast<double2 *>(smem + kSmTwA);
    float *mw = reinterpret_cast<float *>(smem + kSmMelW);
    short *mk = reinterpret_cast<short *>(smem + kSmMelK);
    unsigned char *mb = reinterpret_cast<unsigned char *>(smem + kSmMelB);
    int *ch = reinterpret_cast<int *>(smem + kSmChunk);
    int *sf = reinterpret_cast<int *>(smem + kSmSegFirst);
    int *cs = reinterpret_cast<int *>(smem + kSmChanSeg);
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) w[i] = d_w1600[i];
    for (int i = threadIdx.x; i < 800; i += blockDim.x) {
      h2[i] = d_hann2[i];
      ta[i] = d_twa[i];
    }
    for (int i = threadIdx.x; i < kMelNnzMax; i += blockDim.x) {
      mw[i] = d_melw[i];
      mk[i] = d_melk[i];
      mb[i] = d_melb[i];
    }
    for (int i = threadIdx.x; i < 33; i += blockDim.x) ch[i] = d_chunk[i];
    for (int i = threadIdx.x; i < 33; i += blockDim.x) sf[i] = d_segfirst[i];
    for (int i = threadIdx.x; i < 81; i += blockDim.x) cs[i] = d_chanseg[i];
  }
  __syncthreads();
  const Tables T{reinterpret_cast<const double2 *>(smem + kSmW), reinterpret_cast<const double2 *>(smem + kSmHann),
                 reinterpret_cast<const double2 *>(smem + kSmTwA), reinterpret_cast<const float *>(smem + kSmMelW),
                 reinterpret_cast<const short *>(smem + kSmMelK),
                 reinterpret_cast<const unsigned char *>(smem + kSmMelB), reinterpret_cast<const int *>(smem + kSmChunk),
                 reinterpret_cast<const int *>(smem + kSmSegFirst), reinterpret_cast<const int *>(smem + kSmChanSeg)};
  double2 *B = reinterpret_cast<double2 *>(smem + kSmTables + warp * kWarpBufBytes);
  float *P = reinterpret_cast<float *>(B);  // P (fp32) over the buffer after step D
  float *S = reinterpret_cast<float *>(B);  // the frame's raw samples before step A
  float *part = reinterpret_cast<float *>(smem + kSmTables + warp * kWarpBufBytes + kPartOffset);

  const int64_t warps_total = (int64_t)gridDim.x * kWarpsPerBlock;
  const int64_t gw = (int64_t)blockIdx.x * kWarpsPerBlock + warp;
  const int64_t chunk = (n_frames + warps_total - 1) / warps_total;
  const int64_t g0 = gw * chunk;
  const int64_t g1 = g0 + chunk < n_frames ? g0 + chunk : n_frames;
  if (g0 >= g1) return;

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

  for (int64_t g = g0; g < g1; ++g) {
    while (clip + 1 < n_clips && foff[clip + 1] <= g) ++clip;
    const int64_t t = g - foff[clip];
    const int64_t len = soff[clip + 1] - soff[clip];
    uint8_t *crow = codes + g * kMel;
    if (t < 0 || (int64_t)kHop * (t + 1) > len) {  // offsets do not describe this frame
      if (lane == 0) record_error(err, DMEL_DEVERR_OFFSETS);
      for (int b = lane; b < kMel; b += 32) crow[b] = 0;
      continue;
    }
    // the next frame of this clip needs samples [800 (t + 1), 800 (t + 2)): start them into L1
    if (g + 1 < g1 && (int64_t)kHop * (t + 2) <= len && lane < 25)
      asm volatile("prefetch.global.L1 [%0];" ::"l"(wav + soff[clip] + (int64_t)kHop * (t + 1) + 32 * lane));
    stage_frame(lane, wav + soff[clip], tails ? tails + (int64_t)clip * kHop + kHop : nullptr, (int64_t)kHop * (t - 1),
                S);
    __syncwarp();
    {
      double ar[25], ai[25];
      step_a_load(lane, S, T, ar, ai);
      __syncwarp();  // every lane has its samples before the DFT outputs overwrite them
      step_a_dft(lane, T, ar, ai, B);
    }
    __syncwarp();
    step_c1_lane(lane, T, B);
    __syncwarp();
    step_c2_lane(lane, B);
    __syncwarp();
    {
      PairRegs R;
      step_d_load(lane, B, R);
      __syncwarp();  // every Z value is in registers before P overwrites the buffer
      step_d_store(lane, T, R, P);
    }
    __syncwarp();
    step_e_chunk(lane, T, P, part);
    __syncwarp();
    step_e_codes(lane, T, part, crow, nullptr, qz);
    __syncwarp();
  }
}

// Carried tails: one block per clip row (800 floats); the source is the last 800 consumed
// samples of the clip, or the tail in when the clip has no frame.
__global__ void __launch_bounds__(256) tails_kernel_entry(const float *__restrict__ wav,
                                                          const int64_t *__restrict__ soff,
                                                          const int64_t *__restrict__ foff, int n_clips,
                                                          const float *tails, float *tails_out, uint32_t *err) {
  for (int c = blockIdx.x; c < n_clips; c += gridDim.x) {
    const int64_t F = foff[c + 1] - foff[c];
    const int64_t len = soff[c + 1] - soff[c];
    float *dst = tails_out + (int64_t)c * kHop;
    if (F >= 1 && (int64_t)kHop * F > len) {
      if (threadIdx.x == 0) record_error(err, DMEL_DEVERR_OFFSETS);
      for (int n = threadIdx.x; n < kHop; n += blockDim.x) dst[n] = 0.0f;
      continue;
    }
    const float *src = F >= 1 ? wav + soff[c] + (int64_t)kHop * (F - 1) : (tails ? tails + (int64_t)c * kHop : nullptr);
    if (!src) {
      for (int n = threadIdx.x; n < kHop; n += blockDim.x) dst[n] = 0.0f;
    } else if ((reinterpret_cast<uintptr_t>(src) & 15) == 0 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
      for (int n = threadIdx.x; n < kHop / 4; n += blockDim.x)
        reinterpret_cast<float4 *>(dst)[n] = reinterpret_cast<const float4 *>(src)[n];
    } else {
      for (int n = threadIdx.x; n < kHop; n += blockDim.x) dst[n] = src[n];
    }
  }
}

// ---------------------------------------------------------------- host entry points

cudaError_t launch_codes(const float *wav, const int64_t *soff, const int64_t *foff, int n_clips, int64_t n_frames,
                         const float *tails, float *tails_out, uint8_t *codes, uint32_t *err, int num_sms,
                         cudaStream_t stream, int *launches, Quant q) {
  cudaError_t e = ensure_device_tables();
  if (e != cudaSuccess) return e;
  static std::atomic<bool> attr_set[256];
  if ((e = set_smem_attr_once(codes_kernel_entry, kSmemBytes, attr_set)) != cudaSuccess) return e;
  if (n_frames > 0) {
    int64_t blocks = (n_frames + kWarpsPerBlock - 1) / kWarpsPerBlock;
    if (blocks > num_sms) blocks = num_sms;  // one persistent block per SM
    codes_kernel_entry<<<(unsigned)blocks, kWarpsPerBlock * 32, kSmemBytes, stream>>>(
        wav, soff, foff, n_clips, n_frames, tails, codes, q, err);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ++*launches;
  }
  if (tails_out && n_clips > 0) {
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
  std::vector<PairRegs> R(32);
  std::vector<float> part(kMaxSegs);
  std::vector<double> arb(32 * 25), aib(32 * 25);
  for (int l = 0; l < 32; ++l)
    step_a_load(l, frame1600, T, *reinterpret_cast<double(*)[25]>(&arb[25 * l]),
                *reinterpret_cast<double(*)[25]>(&aib[25 * l]));
  for (int l = 0; l < 32; ++l)
    step_a_dft(l, T, *reinterpret_cast<double(*)[25]>(&arb[25 * l]), *reinterpret_cast<double(*)[25]>(&aib[25 * l]),
               B.data());
  for (int l = 0; l < 32; ++l) step_c1_lane(l, T, B.data());
  for (int l = 0; l < 32; ++l) step_c2_lane(l, B.data());
  for (int l = 0; l < 32; ++l) step_d_load(l, B.data(), R[l]);
  for (int l = 0; l < 32; ++l) step_d_store(l, T, R[l], reinterpret_cast<float *>(B.data()));
  for (int l = 0; l < 32; ++l) step_e_chunk(l, T, reinterpret_cast<const float *>(B.data()), part.data());
  for (int l = 0; l < 32; ++l) step_e_codes(l, T, part.data(), codes80, lhat80, q);
}

}  // namespace dmel
