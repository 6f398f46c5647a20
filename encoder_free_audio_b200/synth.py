"""Seeded synthetic inputs for the dMel front end.

This module only draws signals, tables and codes. It holds none of the front end's arithmetic
(no window, transform, filterbank, quantiser or embedding), so the CUDA path and the CPU oracle
can both be fed from it without sharing any of the method.

Workloads (16 kHz mono fp32, values in [-1, 1]):
  one_clip_2s        one 2 s clip: three sines plus white noise (40 frames)
  batch64_10s        64 clips x 10 s: pink noise plus a linear chirp; 10% of clips silent,
                     5% clipped at +-1 (12,800 frames)
  long_20min         one 20-minute clip of AR(12)-filtered noise bursts with 20% silence
                     (24,000 frames)
  ragged1024         1024 clips of 1..30 s, concatenated with an offsets array, no padding:
                     segments of pink noise, harmonic tones, both, or silence
  streams4096        4096 streams, 800 new samples per stream per call, white noise plus a
                     tone, continuous across calls
Tables are N(0, 0.02) (seed 7), RMSNorm weights N(1, 0.1) (seed 8).
"""
from __future__ import annotations

import numpy as np

SR = 16000
HOP = 800
N_ROWS = 1280
DIM = 6144

SEED_ONE_CLIP = 1001
SEED_BATCH64 = 1002
SEED_LONG = 1003
SEED_RAGGED = 1004
SEED_STREAMS = 1005
SEED_TABLE = 7
SEED_RMS = 8


def _rng(seed) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def pink_noise(rng: np.random.Generator, n: int, rms: float) -> np.ndarray:
    """Gaussian white noise shaped by 1/sqrt(f) in the frequency domain, scaled to `rms`."""
    if n <= 0:
        return np.zeros(0, np.float64)
    spec = np.fft.rfft(rng.standard_normal(n))
    f = np.arange(spec.shape[0], dtype=np.float64)
    f[0] = 1.0
    spec = spec / np.sqrt(f)
    spec[0] = 0.0
    x = np.fft.irfft(spec, n)
    s = np.sqrt(np.mean(x * x))
    return x * (rms / s) if s > 0 else x


def linear_chirp(n: int, f0: float, f1: float, amp: float) -> np.ndarray:
    """amp * cos(2 pi (f0 t + (f1 - f0) t^2 / (2 T))), t in seconds, T the clip duration."""
    t = np.arange(n, dtype=np.float64) / SR
    T = n / SR
    return amp * np.cos(2 * np.pi * (f0 * t + (f1 - f0) * t * t / (2 * T)))


def harmonic_tone(n: int, f0: float, a1: float, n_harm: int = 10, phase0: float = 0.0) -> np.ndarray:
    """sum_{h=1..n_harm} (a1 / h) cos(2 pi h f0 t + h phase0), harmonics above 8 kHz left out."""
    t = np.arange(n, dtype=np.float64) / SR
    x = np.zeros(n, np.float64)
    for h in range(1, n_harm + 1):
        if h * f0 >= SR / 2:
            break
        x += (a1 / h) * np.cos(2 * np.pi * h * f0 * t + h * phase0)
    return x


def offsets_from_lengths(lengths) -> np.ndarray:
    off = np.zeros(len(lengths) + 1, np.int64)
    np.cumsum(np.asarray(lengths, np.int64), out=off[1:])
    return off


# ---------------------------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------------------------

def one_clip_2s(seed: int = SEED_ONE_CLIP):
    """32,000 samples: sum of 3 sines (f ~ U(100, 4000) Hz, A ~ U(0.1, 0.5), phase ~ U(0, 2 pi))
    plus N(0, 0.01^2). Returns (wav fp32 [32000], sample offsets [2])."""
    r = _rng(seed)
    n = 2 * SR
    t = np.arange(n, dtype=np.float64) / SR
    x = np.zeros(n)
    for _ in range(3):
        f, a, ph = r.uniform(100, 4000), r.uniform(0.1, 0.5), r.uniform(0, 2 * np.pi)
        x += a * np.cos(2 * np.pi * f * t + ph)
    x += r.normal(0.0, 0.01, n)
    return x.astype(np.float32), offsets_from_lengths([n])


def batch64_10s(seed: int = SEED_BATCH64, n_clips: int = 64, seconds: float = 10.0):
    """n_clips x 10 s: pink noise (RMS 0.05) + linear chirp 50 -> 7000 Hz (A ~ U(0.1, 0.5));
    10% of clips all zero, 5% scaled x4 then clipped; everything clipped to [-1, 1].
    Returns (wav fp32 [n_clips * 160000], sample offsets [n_clips + 1])."""
    r = _rng(seed)
    n = int(seconds * SR)
    order = r.permutation(n_clips)
    n_sil = int(round(0.10 * n_clips))
    n_clip = int(round(0.05 * n_clips))
    silent = set(order[:n_sil].tolist())
    clipped = set(order[n_sil:n_sil + n_clip].tolist())
    out = np.zeros(n_clips * n, np.float32)
    for c in range(n_clips):
        a = r.uniform(0.1, 0.5)
        x = pink_noise(r, n, 0.05) + linear_chirp(n, 50.0, 7000.0, a)
        if c in silent:
            x[:] = 0.0
        if c in clipped:
            x = 4.0 * x
        out[c * n:(c + 1) * n] = np.clip(x, -1.0, 1.0)
    return out, offsets_from_lengths([n] * n_clips)


def ar12_burst(rng: np.random.Generator, n: int, rms: float) -> np.ndarray:
    """White noise through an all-pole filter with 6 conjugate pole pairs (radius U(0.85, 0.98),
    angle U(0.05 pi, 0.9 pi)), scaled to `rms`."""
    from scipy.signal import lfilter
    rad = rng.uniform(0.85, 0.98, 6)
    ang = rng.uniform(0.05 * np.pi, 0.9 * np.pi, 6)
    poles = np.concatenate([rad * np.exp(1j * ang), rad * np.exp(-1j * ang)])
    a = np.real(np.poly(poles))
    y = lfilter([1.0], a, rng.standard_normal(n))
    s = np.sqrt(np.mean(y * y))
    return y * (rms / s) if s > 0 else y


def long_20min(seed: int = SEED_LONG, n_samples: int = 20 * 60 * SR):
    """One clip of n_samples: bursts of AR(12) noise, 50-400 ms long, RMS U(0.02, 0.3), separated
    by exact-zero gaps drawn so that about 20% of the samples are silence.
    Returns (wav fp32 [n_samples], sample offsets [2])."""
    r = _rng(seed)
    x = np.zeros(n_samples, np.float32)
    pos = 0
    mean_burst = 0.5 * (0.05 + 0.4) * SR
    mean_gap = 0.25 * mean_burst  # gaps / (gaps + bursts) = 0.2
    while pos < n_samples:
        gap = int(r.exponential(mean_gap))
        pos += gap
        if pos >= n_samples:
            break
        nb = int(r.uniform(0.05, 0.4) * SR)
        nb = min(nb, n_samples - pos)
        x[pos:pos + nb] = np.clip(ar12_burst(r, nb, r.uniform(0.02, 0.3)), -1, 1)
        pos += nb
    return x, offsets_from_lengths([n_samples])


def ragged1024(seed: int = SEED_RAGGED, n_clips: int = 1024, min_s: float = 1.0, max_s: float = 30.0,
               workers: int | None = None):
    """n_clips clips with integer lengths uniform in [min_s, max_s] seconds, concatenated without
    padding. Each clip is a run of 0.5-3 s segments, each one of: pink noise (RMS U(0.02, 0.2)),
    a harmonic tone (f0 ~ U(80, 400), 10 harmonics at amplitude a1 / h, a1 ~ U(0.05, 0.4)),
    both, or digital silence. Returns (wav fp32, sample offsets [n_clips + 1]).

    Drawn in bulk so 250M samples take seconds: every segment's parameters first, in clip order;
    the pink noise of a segment is the first samples of a 3 s (48,000-sample) pink-noise draw
    (white noise shaped by 1/sqrt(f), batches of segments per seeded generator), scaled to the
    segment's RMS; the tones are summed through the recurrence
    cos((h+1) u) = 2 cos(u) cos(h u) - cos((h-1) u), u = 2 pi f0 t + phase. Rendering runs on
    `workers` threads over fixed blocks, so the result does not depend on the thread count."""
    from concurrent.futures import ThreadPoolExecutor
    import os
    import scipy.fft as sfft
    r = _rng(seed)
    lengths = r.integers(int(min_s * SR), int(max_s * SR), size=n_clips, endpoint=True)
    off = offsets_from_lengths(lengths)
    total = int(off[-1])
    starts, sizes, kinds, rmss, f0s, a1s, phs = [], [], [], [], [], [], []
    for c in range(n_clips):
        n = int(lengths[c])
        pos = 0
        while pos < n:
            seg = min(int(r.uniform(0.5, 3.0) * SR), n - pos)
            starts.append(int(off[c]) + pos)
            sizes.append(seg)
            kinds.append(int(r.integers(0, 4)))
            rmss.append(r.uniform(0.02, 0.2))
            f0s.append(r.uniform(80, 400))
            a1s.append(r.uniform(0.05, 0.4))
            phs.append(r.uniform(0, 2 * np.pi))
            pos += seg
    starts, sizes, kinds = np.array(starts, np.int64), np.array(sizes, np.int64), np.array(kinds)
    f0s, a1s, phs, rmss = np.array(f0s), np.array(a1s), np.array(phs), np.array(rmss)
    acc = np.zeros(total, np.float64)
    nw = workers or min(16, os.cpu_count() or 1)
    PL = 3 * SR  # longest segment
    pink = np.nonzero((kinds == 0) | (kinds == 2))[0]
    batches = [pink[i:i + 128] for i in range(0, pink.shape[0], 128)]
    fsc = 1.0 / np.sqrt(np.maximum(np.arange(PL // 2 + 1, dtype=np.float64), 1.0))
    fsc[0] = 0.0

    def pink_batch(bi):
        ids = batches[bi]
        g = np.random.Generator(np.random.Philox(key=np.array([seed, bi], np.uint64)))
        x = sfft.irfft(sfft.rfft(g.standard_normal((ids.shape[0], PL), dtype=np.float32), axis=1) * fsc.astype(np.float32),
                       PL, axis=1).astype(np.float64)
        for row, k in enumerate(ids):
            v = x[row, :sizes[k]]
            sd = np.sqrt(np.mean(v * v))
            acc[starts[k]:starts[k] + sizes[k]] = v * (rmss[k] / sd) if sd > 0 else v

    tone = np.nonzero((kinds == 1) | (kinds == 2))[0]
    t_seg = np.repeat(tone, sizes[tone])  # segment of each tone sample, in sample order
    t_pos = np.repeat(starts[tone], sizes[tone])
    t_pos += np.arange(t_pos.shape[0]) - np.repeat(np.cumsum(sizes[tone]) - sizes[tone], sizes[tone])
    BLK = 1 << 21

    def tone_block(bi):
        lo, hi = bi * BLK, min(t_seg.shape[0], (bi + 1) * BLK)
        sid, pos = t_seg[lo:hi], t_pos[lo:hi]
        amp = a1s[sid]
        u = (pos - starts[sid]).astype(np.float64)
        u *= (2 * np.pi / SR) * f0s[sid]
        u += phs[sid]
        c1 = np.cos(u)
        x = c1.copy()
        prev, cur = np.ones_like(c1), c1.copy()
        for h in range(2, 11):  # h f0 <= 4 kHz: every harmonic lies below 8 kHz
            np.multiply(c1, cur, out=u)
            u *= 2.0
            u -= prev
            prev, cur, u = cur, u, prev
            x += cur * (1.0 / h)
        x *= amp
        acc[pos] += x

    with ThreadPoolExecutor(max_workers=nw) as ex:
        list(ex.map(pink_batch, range(len(batches))))
        list(ex.map(tone_block, range((t_seg.shape[0] + BLK - 1) // BLK)))
    wav = np.clip(acc, -1, 1).astype(np.float32)
    return wav, off


class Streams4096:
    """4096 continuous streams; call k supplies samples [800 k, 800 k + 800) of every stream.
    Stream s = A_s cos(2 pi f_s i / 16000 + phi_s) + sigma_s * noise, with f ~ U(100, 4000),
    A ~ U(0.05, 0.5), sigma ~ U(0.001, 0.05). The noise of call k comes from a Philox generator
    keyed by (seed, k), so any call can be regenerated on its own."""

    def __init__(self, seed: int = SEED_STREAMS, n_streams: int = 4096):
        r = _rng(seed)
        self.seed = seed
        self.n = n_streams
        self.f = r.uniform(100, 4000, n_streams)
        self.a = r.uniform(0.05, 0.5, n_streams)
        self.ph = r.uniform(0, 2 * np.pi, n_streams)
        self.sigma = r.uniform(0.001, 0.05, n_streams)

    def call(self, k: int) -> np.ndarray:
        """fp32 [n_streams, 800] of call k (k >= 0)."""
        i = np.arange(HOP * k, HOP * (k + 1), dtype=np.float64)
        tone = self.a[:, None] * np.cos(2 * np.pi * self.f[:, None] * i[None, :] / SR + self.ph[:, None])
        g = np.random.Generator(np.random.Philox(key=np.array([self.seed, k], np.uint64)))
        noise = g.standard_normal((self.n, HOP))
        return np.clip(tone + self.sigma[:, None] * noise, -1, 1).astype(np.float32)


def table(seed: int = SEED_TABLE, rows: int = N_ROWS, dim: int = DIM) -> np.ndarray:
    """fp32 [rows, dim] ~ N(0, 0.02)."""
    return _rng(seed).normal(0.0, 0.02, (rows, dim)).astype(np.float32)


def rms_weight(seed: int = SEED_RMS, dim: int = DIM) -> np.ndarray:
    """fp32 [dim] ~ N(1, 0.1)."""
    return _rng(seed).normal(1.0, 0.1, dim).astype(np.float32)


def random_codes(seed: int, n_frames: int) -> np.ndarray:
    """uint8 [n_frames, 80], uniform over 0..15."""
    return _rng(seed).integers(0, 16, size=(n_frames, 80), dtype=np.uint8)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)
