/*
 * dMel front end: plain, slow CPU oracle in double precision.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load this file:
 * only the test suite, the smoke check and the benchmark's CPU-baseline leg use it.
 *
 * Every step is the plain definition, written out with explicit loops:
 *   framing       "Inside Inkling: Audio Design", Part 1 · Modeling (hop 800, window 1600,
 *                 20 frames per second); causal edge reading, see frame_sample() below
 *   window        periodic Hann (reading; the pages name no window)
 *   DFT + power   naive O(N^2) DFT of size 1600, |X_k|^2 for k = 0..800 (reading)
 *   mel           80 HTK triangles on 0..8000 Hz, no area normalisation (reading;
 *                 Part 1 fixes only "80-channel log-mel")
 *   log/clamp     log10(max(M, 1e-10)) clamped to [-7, 2] (clamp range from Part 1)
 *   quantise      16 equal levels over the clamp range (reading; the Coda says the mapping is
 *                 unpublished, and "Why Thinking Machines Built Inkling Without a Vision
 *                 Encoder" says it is plain rounding with no training)
 *   embedding     sum of the 80 rows 16*b + c_b of a 1280 x D table, optional RMSNorm
 *                 (Part 1: "a frame's 80 rows are summed", "optional RMSNorm")
 *
 * Threads: frames are independent, so the only parallelism is an OpenMP loop over frames.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_SR 16000
#define OR_HOP 800
#define OR_WIN 1600
#define OR_NFFT 1600
#define OR_NBINS 801 /* one-sided bins 0..800 */
#define OR_NMEL 80
#define OR_NLEV 16
#define OR_LMIN (-7.0)
#define OR_LMAX 2.0
#define OR_FLOOR 1e-10

static const double OR_PI = 3.14159265358979323846264338327950288;

int oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Sets the number of threads the frame loops use (n >= 1); returns the number now in effect. */
int oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

/* Frames of one clip: floor(N / hop); negative lengths are an error (-1). */
int64_t oracle_frames_for_length(int64_t n_samples) {
  if (n_samples < 0) return -1;
  return n_samples / OR_HOP;
}

/* Periodic Hann: w[n] = 0.5 - 0.5 cos(2 pi n / 1600). */
void oracle_window(double *w) {
  for (int n = 0; n < OR_WIN; ++n) w[n] = 0.5 - 0.5 * cos(2.0 * OR_PI * (double)n / (double)OR_WIN);
}

/* HTK mel scale and its inverse. */
double oracle_hz_to_mel(double f) { return 2595.0 * log10(1.0 + f / 700.0); }
double oracle_mel_to_hz(double m) { return 700.0 * (pow(10.0, m / 2595.0) - 1.0); }

/* Dense filterbank fb[b * 801 + k] = H_b(10 k Hz): 82 points equally spaced in mel on
 * [0, 8000] Hz, triangle b has its feet at points b and b+2 and its peak (1.0) at b+1. */
void oracle_filterbank(double *fb) {
  double fpts[OR_NMEL + 2];
  const double mtop = oracle_hz_to_mel(OR_SR / 2.0);
  for (int i = 0; i < OR_NMEL + 2; ++i) fpts[i] = oracle_mel_to_hz(mtop * (double)i / (double)(OR_NMEL + 1));
  for (int b = 0; b < OR_NMEL; ++b) {
    const double lo = fpts[b], mid = fpts[b + 1], hi = fpts[b + 2];
    for (int k = 0; k < OR_NBINS; ++k) {
      const double f = 10.0 * (double)k; /* bin k of a 1600-point DFT at 16 kHz */
      const double up = (f - lo) / (mid - lo);
      const double down = (hi - f) / (hi - mid);
      double h = up < down ? up : down;
      if (h < 0.0) h = 0.0;
      fb[b * OR_NBINS + k] = h;
    }
  }
}

/* cos/sin of 2 pi j / 1600 for j = 0..1599, so the DFT below indexes by (k n) mod 1600. */
static double g_cos[OR_NFFT], g_sin[OR_NFFT], g_win[OR_WIN], g_fb[OR_NMEL * OR_NBINS];
static int g_ready = 0;

static void oracle_init(void) {
  if (g_ready) return;
#pragma omp critical(oracle_init_tables)
  {
    if (!g_ready) {
      for (int j = 0; j < OR_NFFT; ++j) {
        g_cos[j] = cos(2.0 * OR_PI * (double)j / (double)OR_NFFT);
        g_sin[j] = sin(2.0 * OR_PI * (double)j / (double)OR_NFFT);
      }
      oracle_window(g_win);
      oracle_filterbank(g_fb);
      g_ready = 1;
    }
  }
}

/* Power spectrum of one raw 1600-sample frame: window, then the naive DFT
 * X_k = sum_n w[n] s[n] exp(-2 pi i k n / 1600), P_k = |X_k|^2, k = 0..800. */
void oracle_power(const double *frame, double *P) {
  oracle_init();
  double u[OR_WIN];
  for (int n = 0; n < OR_WIN; ++n) u[n] = g_win[n] * frame[n];
  for (int k = 0; k < OR_NBINS; ++k) {
    double re = 0.0, im = 0.0;
    int j = 0; /* j = (k n) mod 1600 */
    for (int n = 0; n < OR_NFFT; ++n) {
      re += u[n] * g_cos[j];
      im -= u[n] * g_sin[j];
      j += k;
      if (j >= OR_NFFT) j -= OR_NFFT;
    }
    P[k] = re * re + im * im;
  }
}

/* Mel energies M_b = sum_k H_b(f_k) P_k of one raw frame. */
void oracle_mel(const double *frame, double *M) {
  double P[OR_NBINS];
  oracle_power(frame, P);
  for (int b = 0; b < OR_NMEL; ++b) {
    double acc = 0.0;
    for (int k = 0; k < OR_NBINS; ++k) acc += g_fb[b * OR_NBINS + k] * P[k];
    M[b] = acc;
  }
}

/* L-hat = min(max(log10(max(M, 1e-10)), -7), 2); a NaN energy counts as the floor. */
double oracle_log_clamp(double M) {
  double m = (M > OR_FLOOR) ? M : OR_FLOOR; /* NaN compares false -> floor */
  double L = log10(m);
  if (L < OR_LMIN) L = OR_LMIN;
  if (L > OR_LMAX) L = OR_LMAX;
  return L;
}

/* 16 equal levels over [-7, 2]: c = min(15, floor((L-hat + 7) * 16 / 9)). */
int oracle_quantise(double lhat) {
  const double q = floor((lhat - OR_LMIN) * (double)OR_NLEV / (OR_LMAX - OR_LMIN));
  int c = (int)q;
  if (c > OR_NLEV - 1) c = OR_NLEV - 1;
  if (c < 0) c = 0;
  return c;
}

/* Sample i of clip `clip` relative to its start, for -800 <= i < N: negative indices read the
 * carried tail (tails[clip * 800 + 800 + i]) or zero without one. */
static double frame_sample(const float *wav, const int64_t *soff, const float *tails, int clip, int64_t i) {
  if (i >= 0) return (double)wav[soff[clip] + i];
  if (!tails) return 0.0;
  return (double)tails[(int64_t)clip * OR_HOP + OR_HOP + i];
}

/* Frame offsets: fo[0] = 0, fo[c+1] = fo[c] + floor((soff[c+1] - soff[c]) / 800).
 * Returns 0, or -1 when the sample offsets do not start at 0 or decrease. */
int oracle_frame_offsets(const int64_t *soff, int n_clips, int64_t *fo) {
  if (n_clips < 0 || soff[0] != 0) return -1;
  fo[0] = 0;
  for (int c = 0; c < n_clips; ++c) {
    const int64_t n = soff[c + 1] - soff[c];
    if (n < 0) return -1;
    fo[c + 1] = fo[c] + oracle_frames_for_length(n);
  }
  return 0;
}

/* Codes for a list of global frame indices (frame_ids == NULL means all frames in order).
 * codes[i * 80 + b], and, when lhat != NULL, the clamped pre-quantisation value
 * lhat[i * 80 + b]. Returns 0, or -1 on bad offsets / frame index. */
int oracle_codes(const float *wav, const int64_t *soff, int n_clips, const float *tails, const int64_t *frame_ids,
                 int64_t n_sel, uint8_t *codes, double *lhat) {
  oracle_init();
  int64_t *fo = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_clips + 1));
  if (!fo) return -1;
  if (oracle_frame_offsets(soff, n_clips, fo) != 0) { free(fo); return -1; }
  const int64_t total = fo[n_clips];
  if (!frame_ids) n_sel = total;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(| : bad)
  for (int64_t i = 0; i < n_sel; ++i) {
    const int64_t g = frame_ids ? frame_ids[i] : i;
    if (g < 0 || g >= total) { bad |= 1; continue; }
    /* clip holding global frame g: the last clip with fo[clip] <= g, so fo[clip+1] > g */
    int lo = 0, hi = n_clips - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) / 2;
      if (fo[mid] <= g) lo = mid; else hi = mid - 1;
    }
    const int64_t t = g - fo[lo];
    double frame[OR_WIN], M[OR_NMEL];
    for (int n = 0; n < OR_WIN; ++n) frame[n] = frame_sample(wav, soff, tails, lo, OR_HOP * (t - 1) + n);
    oracle_mel(frame, M);
    for (int b = 0; b < OR_NMEL; ++b) {
      const double L = oracle_log_clamp(M[b]);
      codes[i * OR_NMEL + b] = (uint8_t)oracle_quantise(L);
      if (lhat) lhat[i * OR_NMEL + b] = L;
    }
  }
  free(fo);
  return bad ? -1 : 0;
}

/* ---- Quantiser variants. The pages leave the level mapping open ("Inside Inkling: Audio
 * Design", Coda: the quantizer mapping is undocumented, uniform or mu-law or learned, and the
 * serving default clamps at -1.5 where the released config says -7.0). With the log-mel value
 * clamped to [lmin, lmax] and u = (L - lmin) / (lmax - lmin):
 *   mode 0, uniform floor (the default reading): c = min(15, floor((L - lmin) * 16 / (lmax - lmin)))
 *   mode 1, nearest of the 16 reconstruction points lmin + k (lmax - lmin) / 15, ties upward:
 *           c = floor((L - lmin) * 15 / (lmax - lmin) + 1/2)
 *   mode 2, mu-law companding then 16 uniform levels: c = min(15, floor(16 ln(1 + mu u) / ln(1 + mu)))
 * Codes always end in 0..15. */
double oracle_log_clamp_q(double M, double lmin, double lmax) {
  double m = (M > OR_FLOOR) ? M : OR_FLOOR; /* NaN compares false -> floor */
  double L = log10(m);
  if (L < lmin) L = lmin;
  if (L > lmax) L = lmax;
  return L;
}

int oracle_quantise_q(double lhat, double lmin, double lmax, int mode, double mu) {
  double q;
  if (mode == 1) {
    q = floor((lhat - lmin) * (double)(OR_NLEV - 1) / (lmax - lmin) + 0.5);
  } else if (mode == 2) {
    const double u = (lhat - lmin) / (lmax - lmin);
    q = floor((double)OR_NLEV * log(1.0 + mu * u) / log(1.0 + mu));
  } else {
    q = floor((lhat - lmin) * (double)OR_NLEV / (lmax - lmin));
  }
  int c = (int)q;
  if (c > OR_NLEV - 1) c = OR_NLEV - 1;
  if (c < 0) c = 0;
  return c;
}

/* oracle_codes with a quantiser variant; lhat receives the value clamped to [lmin, lmax]. */
int oracle_codes_q(const float *wav, const int64_t *soff, int n_clips, const float *tails, const int64_t *frame_ids,
                   int64_t n_sel, double lmin, double lmax, int mode, double mu, uint8_t *codes, double *lhat) {
  oracle_init();
  int64_t *fo = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_clips + 1));
  if (!fo) return -1;
  if (oracle_frame_offsets(soff, n_clips, fo) != 0) { free(fo); return -1; }
  const int64_t total = fo[n_clips];
  if (!frame_ids) n_sel = total;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(| : bad)
  for (int64_t i = 0; i < n_sel; ++i) {
    const int64_t g = frame_ids ? frame_ids[i] : i;
    if (g < 0 || g >= total) { bad |= 1; continue; }
    int lo = 0, hi = n_clips - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) / 2;
      if (fo[mid] <= g) lo = mid; else hi = mid - 1;
    }
    const int64_t t = g - fo[lo];
    double frame[OR_WIN], M[OR_NMEL];
    for (int n = 0; n < OR_WIN; ++n) frame[n] = frame_sample(wav, soff, tails, lo, OR_HOP * (t - 1) + n);
    oracle_mel(frame, M);
    for (int b = 0; b < OR_NMEL; ++b) {
      const double L = oracle_log_clamp_q(M[b], lmin, lmax);
      codes[i * OR_NMEL + b] = (uint8_t)oracle_quantise_q(L, lmin, lmax, mode, mu);
      if (lhat) lhat[i * OR_NMEL + b] = L;
    }
  }
  free(fo);
  return bad ? -1 : 0;
}

/* Carried tails out: the 800 samples that end at sample 800 F of each clip (F >= 1), else the
 * tail in (zeros without one). */
int oracle_tails_out(const float *wav, const int64_t *soff, int n_clips, const float *tails, float *tails_out) {
  for (int c = 0; c < n_clips; ++c) {
    const int64_t F = oracle_frames_for_length(soff[c + 1] - soff[c]);
    if (F < 0) return -1;
    for (int n = 0; n < OR_HOP; ++n)
      tails_out[(int64_t)c * OR_HOP + n] = (float)frame_sample(wav, soff, tails, c, OR_HOP * F - OR_HOP + n);
  }
  return 0;
}

/* Embedding of frames: x_j = sum_b T[16 b + c_b, j] in double; with g != NULL,
 * y_j = g_j x_j / sqrt(mean_j x_j^2 + eps). table is [1280 x dim] row-major. */
int oracle_embed(const uint8_t *codes, int64_t n_frames, const double *table, int dim, const double *g, double eps,
                 double *out) {
  if (dim <= 0 || n_frames < 0) return -1;
  int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
  for (int64_t f = 0; f < n_frames; ++f) {
    double *y = out + f * (int64_t)dim;
    for (int j = 0; j < dim; ++j) y[j] = 0.0;
    for (int b = 0; b < OR_NMEL; ++b) {
      const int c = codes[f * OR_NMEL + b];
      if (c >= OR_NLEV) { bad |= 1; continue; }
      const double *row = table + (int64_t)(OR_NLEV * b + c) * dim;
      for (int j = 0; j < dim; ++j) y[j] += row[j];
    }
    if (g) {
      double ss = 0.0;
      for (int j = 0; j < dim; ++j) ss += y[j] * y[j];
      const double inv = 1.0 / sqrt(ss / (double)dim + eps);
      for (int j = 0; j < dim; ++j) y[j] = g[j] * (y[j] * inv);
    }
  }
  return bad ? -1 : 0;
}

/* ---- ShortConv ("Inside Inkling: Audio Design", Part 3 · Inference): per-channel causal
 * convolution of width W = 4 with the input added back,
 *     y[t, c] = x[t, c] + sum_{d=0}^{3} w[c, d] * x[t - d, c],
 * over each sequence s of tokens [off[s], off[s+1]). Inputs before a sequence's first token
 * come from its carried state (state[s][3 + j] = x[j] for j = -3, -2, -1; all zero without a
 * state). state_out[s] receives the last three inputs the sequence ends with (taking them from
 * the state in when the sequence is shorter than three). Everything in fp64. */
int oracle_shortconv(const double *x, const int64_t *off, int n_seq, int C, const double *w, const double *state,
                     double *y, double *state_out) {
  for (int s = 0; s < n_seq; ++s) {
    const int64_t t0 = off[s], T = off[s + 1] - off[s];
    if (T < 0) return -1;
    for (int64_t t = 0; t < T; ++t)
      for (int c = 0; c < C; ++c) {
        double acc = x[(t0 + t) * C + c];
        for (int d = 0; d < 4; ++d) {
          const int64_t j = t - d;
          double xv;
          if (j >= 0) xv = x[(t0 + j) * C + c];
          else xv = state ? state[((int64_t)s * 3 + 3 + j) * C + c] : 0.0;
          acc += w[c * 4 + d] * xv;
        }
        y[(t0 + t) * C + c] = acc;
      }
    if (state_out)
      for (int i = 0; i < 3; ++i) {
        const int64_t j = T - 3 + i; /* position of state row i relative to the sequence start */
        for (int c = 0; c < C; ++c) {
          double v;
          if (j >= 0) v = x[(t0 + j) * C + c];
          else v = state ? state[((int64_t)s * 3 + 3 + j) * C + c] : 0.0;
          state_out[((int64_t)s * 3 + i) * C + c] = v;
        }
      }
  }
  return 0;
}
