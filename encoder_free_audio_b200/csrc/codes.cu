// dMel codes: framing, periodic Hann window, 1600-point DFT power, 80 HTK mel channels,
// log10, clamp to [-7, 2], 16 equal levels ("Inside Inkling: Audio Design", Part 1 · Modeling;
// the window, DFT size, mel formula, log base/floor and level boundaries are this library's
// readings of what the pages leave open, stated in include/dmel.h).
//
// One warp computes one frame; a warp walks a contiguous run of frames so that consecutive
// frames share half their samples through L1. The transform runs in fp64 so that the codes
// agree with an exact evaluation everywhere except within ~1e-12 of a level boundary.
//
// Real DFT of 1600 points through one complex DFT of 800 points, z_m = u_{2m} + i u_{2m+1}
// (u = windowed samples), 800 = 25 x 32:
//   A  lane l (0..31) takes z_{32 j + l}, j = 0..24, does a 25-point DFT in registers (5 x 5),
//      multiplies output k1 by W_800^{l k1} and writes Y[k1][l];
//   C  lane k1 (0..24) takes Y[k1][0..31], does a 32-point DFT (radix 2) and writes
//      Z[k1 + 25 k2];
//   D  X_k = (Z_k + conj Z_{800-k}) / 2 + W_1600^k (Z_k - conj Z_{800-k}) / (2 i), P_k = |X_k|^2;
//   E  lane l sums the sparse mel triangles assigned to it, then log10, clamp, quantise.
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace dmel {
namespace {

constexpr int kYStride = 33;                 // padded row of Y[25][33] (bank spread)
constexpr int kYElems = 25 * kYStride;       // 825 complex values; P[801] reuses this space
constexpr int kZElems = 800;
constexpr int kWarpSmemBytes = (kYElems + kZElems) * 16;  // 26,000 B per warp
constexpr int kWarpsPerBlock = 4;
constexpr int kMaxFiltPerLane = 8;
constexpr int kMelNnzMax = 2048;

// Constant tables, filled once per device from host-computed fp64 values.
__device__ double d_win[kWin];
__device__ double2 d_w800[800];
__device__ double2 d_w1600[kBins];
__device__ double d_melw[kMelNnzMax];
__device__ int d_mel_k0[kMel];
__device__ int d_mel_n[kMel];
__device__ int d_mel_off[kMel];
__device__ signed char d_lane_filt[32 * kMaxFiltPerLane];

struct Tables {
  const double *win;
  const double2 *w800;
  const double2 *w1600;
  const double *melw;
  const int *mel_k0;
  const int *mel_n;
  const int *mel_off;
  const signed char *lane_filt;
};

__host__ __device__ inline void cmul(double &re, double &im, double wr, double wi) {
  const double r = re * wr - im * wi;
  const double i = re * wi + im * wr;
  re = r;
  im = i;
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

// Raw sample n (0..1599) of frame t of a clip: x[800 (t - 1) + n], with samples before the clip
// taken from the carried tail (tail points one past its last sample) or zero.
struct ClipSampler {
  const float *base;
  const float *tail;
  int64_t start;
  __host__ __device__ double operator()(int n) const {
    const int64_t i = start + n;
    if (i >= 0) return (double)base[i];
    return tail ? (double)tail[i] : 0.0;
  }
};

// Sample n of one already-framed 1600-sample buffer.
struct FrameSampler {
  const float *frame;
  __host__ __device__ double operator()(int n) const { return (double)frame[n]; }
};

__host__ __device__ inline int bitrev5(int k) {
  return ((k & 1) << 4) | ((k & 2) << 2) | (k & 4) | ((k & 8) >> 2) | ((k & 16) >> 4);
}

// Step A for lane l. sample(n) returns raw frame sample n (0..1599) as double.
template <class SampleFn>
__host__ __device__ inline void step_a(int l, SampleFn sample, const Tables &T, double2 *Y) {
  double ar[25], ai[25];
#pragma unroll
  for (int j = 0; j < 25; ++j) {
    const int n0 = 64 * j + 2 * l;
    ar[j] = T.win[n0] * sample(n0);
    ai[j] = T.win[n0 + 1] * sample(n0 + 1);
  }
  // 25 = 5 x 5, j = j1 + 5 j2: inner DFTs over j2, result for (j1, ka) stored at j1 + 5 ka
#pragma unroll
  for (int j1 = 0; j1 < 5; ++j1)
    dft5(ar[j1], ai[j1], ar[j1 + 5], ai[j1 + 5], ar[j1 + 10], ai[j1 + 10], ar[j1 + 15], ai[j1 + 15], ar[j1 + 20],
         ai[j1 + 20]);
  // twiddle W_25^{j1 ka} = W_800^{32 j1 ka}
#pragma unroll
  for (int j1 = 1; j1 < 5; ++j1)
#pragma unroll
    for (int ka = 1; ka < 5; ++ka) {
      const double2 w = T.w800[(32 * j1 * ka) % 800];
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
      if (l * k1 != 0) {
        const double2 w = T.w800[(l * k1) % 800];  // W_800^{l k1}
        cmul(yr, yi, w.x, w.y);
      }
      Y[k1 * kYStride + l] = make_double2(yr, yi);
    }
  }
}

// Step C for lane k1 < 25: 32-point DFT over l of Y[k1][l], written to Z[k1 + 25 k2].
__host__ __device__ inline void step_c(int k1, const Tables &T, const double2 *Y, double2 *Z) {
  double re[32], im[32];
#pragma unroll
  for (int l = 0; l < 32; ++l) {
    const double2 y = Y[k1 * kYStride + l];
    re[l] = y.x;
    im[l] = y.y;
  }
  // radix-2 decimation in frequency; output k lands at position bitrev5(k)
#pragma unroll
  for (int span = 16; span >= 1; span >>= 1) {
#pragma unroll
    for (int start = 0; start < 32; start += 2 * span) {
#pragma unroll
      for (int i = 0; i < span; ++i) {
        const int a = start + i, b = a + span;
        const double tr = re[a] - re[b], ti = im[a] - im[b];
        re[a] += re[b];
        im[a] += im[b];
        const int m = i * (16 / span);  // W_{2 span}^i = W_32^m = W_800^{25 m}
        if (m == 0) {
          re[b] = tr;
          im[b] = ti;
        } else {
          const double2 w = T.w800[25 * m];
          re[b] = tr * w.x - ti * w.y;
          im[b] = tr * w.y + ti * w.x;
        }
      }
    }
  }
#pragma unroll
  for (int k2 = 0; k2 < 32; ++k2) {
    const int p = bitrev5(k2);
    Z[k1 + 25 * k2] = make_double2(re[p], im[p]);
  }
}

// Step D for lane l: power of bins k = l, l + 32, ... <= 800.
__host__ __device__ inline void step_d(int l, const Tables &T, const double2 *Z, double *P) {
  for (int k = l; k <= 800; k += 32) {
    const double2 a = Z[k % 800];
    const double2 b = Z[(800 - k) % 800];
    const double er = 0.5 * (a.x + b.x), ei = 0.5 * (a.y - b.y);  // (Z_k + conj Z_{800-k}) / 2
    const double dr = a.x - b.x, di = a.y + b.y;                    // Z_k - conj Z_{800-k}
    const double or_ = 0.5 * di, oi = -0.5 * dr;                    // / (2 i)
    const double2 w = T.w1600[k];
    const double xr = er + (or_ * w.x - oi * w.y);
    const double xi = ei + (or_ * w.y + oi * w.x);
    P[k] = xr * xr + xi * xi;
  }
}

// Step E for lane l: mel channels assigned to this lane -> clamped log10 and level.
__host__ __device__ inline void step_e(int l, const Tables &T, const double *P, uint8_t *codes_row, double *lhat_row) {
  for (int s = 0; s < kMaxFiltPerLane; ++s) {
    const int b = T.lane_filt[l * kMaxFiltPerLane + s];
    if (b < 0) break;
    const int k0 = T.mel_k0[b], n = T.mel_n[b], off = T.mel_off[b];
    double acc = 0.0;
    for (int i = 0; i < n; ++i) acc += T.melw[off + i] * P[k0 + i];
    double L = log10(fmax(acc, 1e-10));  // fmax drops a NaN energy
    L = fmin(fmax(L, -7.0), 2.0);
    int c = (int)floor((L + 7.0) * 16.0 / 9.0);
    c = c > 15 ? 15 : (c < 0 ? 0 : c);
    codes_row[b] = (uint8_t)c;
    if (lhat_row) lhat_row[b] = L;
  }
}

// ---------------------------------------------------------------- host tables

struct HostTables {
  std::vector<double> win, melw;
  std::vector<double2> w800, w1600;
  int k0[kMel], n[kMel], off[kMel];
  signed char lane_filt[32 * kMaxFiltPerLane];
  Tables view() const {
    return Tables{win.data(), w800.data(), w1600.data(), melw.data(), k0, n, off, lane_filt};
  }
};

void build_host_tables(HostTables &H) {
  const double two_pi = 6.283185307179586476925286766559;
  H.win.resize(kWin);
  for (int i = 0; i < kWin; ++i) H.win[i] = 0.5 - 0.5 * std::cos(two_pi * i / kWin);
  H.w800.resize(800);
  for (int j = 0; j < 800; ++j) H.w800[j] = make_double2(std::cos(two_pi * j / 800), -std::sin(two_pi * j / 800));
  H.w1600.resize(kBins);
  for (int k = 0; k < kBins; ++k)
    H.w1600[k] = make_double2(std::cos(two_pi * k / 1600), -std::sin(two_pi * k / 1600));
  // HTK mel points: 82 points equally spaced in mel on [0, 8000] Hz
  const double mel_top = 2595.0 * std::log10(1.0 + 8000.0 / 700.0);
  double fp[kMel + 2];
  for (int i = 0; i < kMel + 2; ++i) fp[i] = 700.0 * (std::pow(10.0, (mel_top * i / (kMel + 1)) / 2595.0) - 1.0);
  H.melw.clear();
  for (int b = 0; b < kMel; ++b) {
    H.off[b] = (int)H.melw.size();
    H.k0[b] = -1;
    H.n[b] = 0;
    for (int k = 0; k < kBins; ++k) {
      const double f = 10.0 * k;
      const double up = (f - fp[b]) / (fp[b + 1] - fp[b]);
      const double down = (fp[b + 2] - f) / (fp[b + 2] - fp[b + 1]);
      const double h = up < down ? up : down;
      if (h > 0.0) {
        if (H.k0[b] < 0) H.k0[b] = k;
        H.melw.push_back(h);
        ++H.n[b];
      }
    }
  }
  // longest-first assignment of channels to lanes, balancing summed triangle widths
  int load[32] = {0}, cnt[32] = {0};
  std::memset(H.lane_filt, -1, sizeof(H.lane_filt));
  int order[kMel];
  for (int b = 0; b < kMel; ++b) order[b] = b;
  for (int a = 0; a < kMel; ++a)
    for (int c = a + 1; c < kMel; ++c)
      if (H.n[order[c]] > H.n[order[a]]) std::swap(order[a], order[c]);
  for (int a = 0; a < kMel; ++a) {
    int best = 0;
    for (int l = 1; l < 32; ++l)
      if (cnt[l] < kMaxFiltPerLane && (load[l] < load[best] || cnt[best] >= kMaxFiltPerLane)) best = l;
    H.lane_filt[best * kMaxFiltPerLane + cnt[best]++] = (signed char)order[a];
    load[best] += H.n[order[a]];
  }
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
  if ((e = cudaMemcpyToSymbol(d_win, H.win.data(), sizeof(double) * kWin)) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_w800, H.w800.data(), sizeof(double2) * 800)) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_w1600, H.w1600.data(), sizeof(double2) * kBins)) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_melw, H.melw.data(), sizeof(double) * H.melw.size())) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_mel_k0, H.k0, sizeof(H.k0))) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_mel_n, H.n, sizeof(H.n))) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_mel_off, H.off, sizeof(H.off))) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_lane_filt, H.lane_filt, sizeof(H.lane_filt))) != cudaSuccess) return e;
  g_uploaded[dev] = true;
  return cudaSuccess;
}

}  // namespace

// ---------------------------------------------------------------- kernels

__global__ void __launch_bounds__(kWarpsPerBlock * 32) codes_kernel_entry(const float *__restrict__ wav,
                                                                          const int64_t *__restrict__ soff,
                                                                          const int64_t *__restrict__ foff, int n_clips,
                                                                          int64_t n_frames,
                                                                          const float *__restrict__ tails,
                                                                          uint8_t *__restrict__ codes, uint32_t *err) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  double2 *Y = reinterpret_cast<double2 *>(smem + warp * kWarpSmemBytes);
  double2 *Z = Y + kYElems;
  double *P = reinterpret_cast<double *>(Y);  // Y is dead once step C has run
  const Tables T{d_win, d_w800, d_w1600, d_melw, d_mel_k0, d_mel_n, d_mel_off, d_lane_filt};

  const int64_t warps_total = (int64_t)gridDim.x * kWarpsPerBlock;
  const int64_t gw = (int64_t)blockIdx.x * kWarpsPerBlock + warp;
  const int64_t chunk = (n_frames + warps_total - 1) / warps_total;
  const int64_t g0 = gw * chunk;
  const int64_t g1 = g0 + chunk < n_frames ? g0 + chunk : n_frames;
  if (g0 >= g1) return;

  // last clip with foff[clip] <= g0
  int lo = 0, hi = n_clips - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (foff[mid] <= g0) lo = mid; else hi = mid - 1;
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
    const ClipSampler sample{wav + soff[clip], tails ? tails + (int64_t)clip * kHop + kHop : nullptr,
                             (int64_t)kHop * (t - 1)};
    step_a(lane, sample, T, Y);
    __syncwarp();
    if (lane < 25) step_c(lane, T, Y, Z);
    __syncwarp();
    step_d(lane, T, Z, P);
    __syncwarp();
    step_e(lane, T, P, crow, nullptr);
    __syncwarp();
  }
}

__global__ void tails_kernel_entry(const float *__restrict__ wav, const int64_t *__restrict__ soff,
                                   const int64_t *__restrict__ foff, int n_clips, const float *tails,
                                   float *tails_out, uint32_t *err) {
  const int64_t total = (int64_t)n_clips * kHop;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(idx / kHop);
    const int n = (int)(idx % kHop);
    const int64_t F = foff[c + 1] - foff[c];
    const int64_t len = soff[c + 1] - soff[c];
    float v;
    if (F >= 1) {
      if ((int64_t)kHop * F <= len) {
        v = wav[soff[c] + (int64_t)kHop * (F - 1) + n];
      } else {
        record_error(err, DMEL_DEVERR_OFFSETS);
        v = 0.0f;
      }
    } else {
      v = tails ? tails[idx] : 0.0f;
    }
    tails_out[idx] = v;
  }
}

// ---------------------------------------------------------------- host entry points

cudaError_t launch_codes(const float *wav, const int64_t *soff, const int64_t *foff, int n_clips, int64_t n_frames,
                         const float *tails, float *tails_out, uint8_t *codes, uint32_t *err, int num_sms,
                         cudaStream_t stream, int *launches) {
  cudaError_t e = ensure_device_tables();
  if (e != cudaSuccess) return e;
  static bool attr_set[256] = {false};
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (!attr_set[dev & 255]) {
    e = cudaFuncSetAttribute(codes_kernel_entry, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kWarpSmemBytes * kWarpsPerBlock);
    if (e != cudaSuccess) return e;
    attr_set[dev & 255] = true;
  }
  if (n_frames > 0) {
    int64_t blocks = (n_frames + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int64_t cap = (int64_t)num_sms * 2;
    if (blocks > cap) blocks = cap;
    codes_kernel_entry<<<(unsigned)blocks, kWarpsPerBlock * 32, kWarpSmemBytes * kWarpsPerBlock, stream>>>(
        wav, soff, foff, n_clips, n_frames, tails, codes, err);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ++*launches;
  }
  if (tails_out && n_clips > 0) {
    const int64_t total = (int64_t)n_clips * kHop;
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    tails_kernel_entry<<<(unsigned)blocks, 256, 0, stream>>>(wav, soff, foff, n_clips, tails, tails_out, err);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ++*launches;
  }
  return cudaSuccess;
}

// Host emulation of the per-frame arithmetic of codes_kernel_entry (the same step functions,
// lanes run one after another). Diagnostic only: no entry point of the front end calls it.
void emulate_codes_frame_host(const float *frame1600, uint8_t *codes80, double *lhat80) {
  const HostTables &H = host_tables();
  const Tables T = H.view();
  std::vector<double2> Yb(kYElems), Zb(kZElems);
  std::vector<double> Pb(kBins);
  const FrameSampler sample{frame1600};
  for (int l = 0; l < 32; ++l) step_a(l, sample, T, Yb.data());
  for (int l = 0; l < 25; ++l) step_c(l, T, Yb.data(), Zb.data());
  for (int l = 0; l < 32; ++l) step_d(l, T, Zb.data(), Pb.data());
  for (int l = 0; l < 32; ++l) step_e(l, T, Pb.data(), codes80, lhat80);
}

}  // namespace dmel
