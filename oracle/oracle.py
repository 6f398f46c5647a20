"""Python face of the CPU oracle (``dmel_oracle.c``): build it with gcc, load it with ctypes.

TEST INFRASTRUCTURE ONLY. The test suite, the smoke check and the benchmark's CPU-baseline
leg may use this module; the product package never imports it.

Each function states the step it computes; the C file cites the passage each step follows
("Inside Inkling: Audio Design", Part 1 · Modeling, and the readings listed there).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dmel_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")

HOP = 800
WIN = 1600
NBINS = 801
NMEL = 80
NLEV = 16
LMIN = -7.0
LMAX = 2.0

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle (plain -O2, no fast-math) into oracle/_build/liboracle.so."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
               "-std=c11", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        c_d, c_i64, c_int = ctypes.c_double, ctypes.c_int64, ctypes.c_int
        vp = ctypes.c_void_p
        L.oracle_threads.restype = c_int
        L.oracle_set_threads.argtypes = [c_int]
        L.oracle_set_threads.restype = c_int
        L.oracle_frames_for_length.argtypes = [c_i64]
        L.oracle_frames_for_length.restype = c_i64
        L.oracle_window.argtypes = [vp]
        L.oracle_hz_to_mel.argtypes = [c_d]
        L.oracle_hz_to_mel.restype = c_d
        L.oracle_mel_to_hz.argtypes = [c_d]
        L.oracle_mel_to_hz.restype = c_d
        L.oracle_filterbank.argtypes = [vp]
        L.oracle_power.argtypes = [vp, vp]
        L.oracle_mel.argtypes = [vp, vp]
        L.oracle_log_clamp.argtypes = [c_d]
        L.oracle_log_clamp.restype = c_d
        L.oracle_quantise.argtypes = [c_d]
        L.oracle_quantise.restype = c_int
        L.oracle_frame_offsets.argtypes = [vp, c_int, vp]
        L.oracle_frame_offsets.restype = c_int
        L.oracle_codes.argtypes = [vp, vp, c_int, vp, vp, c_i64, vp, vp]
        L.oracle_codes.restype = c_int
        L.oracle_tails_out.argtypes = [vp, vp, c_int, vp, vp]
        L.oracle_tails_out.restype = c_int
        L.oracle_log_clamp_q.argtypes = [c_d, c_d, c_d]
        L.oracle_log_clamp_q.restype = c_d
        L.oracle_quantise_q.argtypes = [c_d, c_d, c_d, c_int, c_d]
        L.oracle_quantise_q.restype = c_int
        L.oracle_codes_q.argtypes = [vp, vp, c_int, vp, vp, c_i64, c_d, c_d, c_int, c_d, vp, vp]
        L.oracle_codes_q.restype = c_int
        L.oracle_shortconv.argtypes = [vp, vp, c_int, c_int, vp, vp, vp, vp]
        L.oracle_shortconv.restype = c_int
        L.oracle_embed.argtypes = [vp, c_i64, vp, c_int, vp, c_d, vp]
        L.oracle_embed.restype = c_int
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def threads() -> int:
    """OpenMP threads the oracle's frame loops use."""
    return int(lib().oracle_threads())


def set_threads(n: int) -> int:
    """Sets the OpenMP threads of the frame loops (n >= 1); returns the count now in effect."""
    return int(lib().oracle_set_threads(int(n)))


def frames_for_length(n: int) -> int:
    """floor(n / 800): frames of an n-sample clip (-1 for n < 0)."""
    return int(lib().oracle_frames_for_length(int(n)))


def window() -> np.ndarray:
    """Periodic Hann window of 1600 points."""
    w = np.zeros(WIN, np.float64)
    lib().oracle_window(_ptr(w))
    return w


def hz_to_mel(f: float) -> float:
    return float(lib().oracle_hz_to_mel(float(f)))


def mel_to_hz(m: float) -> float:
    return float(lib().oracle_mel_to_hz(float(m)))


def filterbank() -> np.ndarray:
    """[80, 801] HTK triangular filterbank evaluated at 10 Hz bin spacing."""
    fb = np.zeros((NMEL, NBINS), np.float64)
    lib().oracle_filterbank(_ptr(fb))
    return fb


def power(frame: np.ndarray) -> np.ndarray:
    """|DFT(window * frame)|^2 for bins 0..800 of one raw 1600-sample frame (naive DFT)."""
    fr = np.ascontiguousarray(frame, np.float64)
    assert fr.shape == (WIN,)
    P = np.zeros(NBINS, np.float64)
    lib().oracle_power(_ptr(fr), _ptr(P))
    return P


def mel(frame: np.ndarray) -> np.ndarray:
    """80 mel energies of one raw 1600-sample frame."""
    fr = np.ascontiguousarray(frame, np.float64)
    assert fr.shape == (WIN,)
    M = np.zeros(NMEL, np.float64)
    lib().oracle_mel(_ptr(fr), _ptr(M))
    return M


def log_clamp(M: float) -> float:
    """min(max(log10(max(M, 1e-10)), -7), 2)."""
    return float(lib().oracle_log_clamp(float(M)))


def quantise(lhat: float) -> int:
    """min(15, floor((lhat + 7) * 16 / 9))."""
    return int(lib().oracle_quantise(float(lhat)))


def frame_offsets(sample_offsets: np.ndarray) -> np.ndarray:
    so = np.ascontiguousarray(sample_offsets, np.int64)
    n = so.shape[0] - 1
    fo = np.zeros(n + 1, np.int64)
    rc = lib().oracle_frame_offsets(_ptr(so), n, _ptr(fo))
    if rc != 0:
        raise ValueError("bad sample offsets")
    return fo


def codes(wav: np.ndarray, sample_offsets: np.ndarray, tails: np.ndarray | None = None,
          frame_ids: np.ndarray | None = None, want_lhat: bool = True):
    """dMel codes [n, 80] (uint8) and clamped log-mel values [n, 80] (float64) for all frames
    (frame_ids None) or for the listed global frame indices."""
    w = np.ascontiguousarray(wav, np.float32)
    so = np.ascontiguousarray(sample_offsets, np.int64)
    n_clips = so.shape[0] - 1
    t = None if tails is None else np.ascontiguousarray(tails, np.float32)
    if t is not None:
        assert t.shape == (n_clips, HOP)
    if frame_ids is None:
        n = int(frame_offsets(so)[-1])
        ids = None
    else:
        ids = np.ascontiguousarray(frame_ids, np.int64)
        n = ids.shape[0]
    c = np.zeros((n, NMEL), np.uint8)
    lh = np.zeros((n, NMEL), np.float64) if want_lhat else None
    rc = lib().oracle_codes(_ptr(w), _ptr(so), n_clips, _ptr(t), _ptr(ids), n, _ptr(c), _ptr(lh))
    if rc != 0:
        raise ValueError("oracle_codes: bad offsets or frame index")
    return (c, lh) if want_lhat else c


def tails_out(wav: np.ndarray, sample_offsets: np.ndarray, tails: np.ndarray | None = None) -> np.ndarray:
    """Carried tail after each clip: the 800 samples ending at sample 800 * F."""
    w = np.ascontiguousarray(wav, np.float32)
    so = np.ascontiguousarray(sample_offsets, np.int64)
    n_clips = so.shape[0] - 1
    t = None if tails is None else np.ascontiguousarray(tails, np.float32)
    out = np.zeros((n_clips, HOP), np.float32)
    rc = lib().oracle_tails_out(_ptr(w), _ptr(so), n_clips, _ptr(t), _ptr(out))
    if rc != 0:
        raise ValueError("bad sample offsets")
    return out


def embed(codes_: np.ndarray, table: np.ndarray, rms_weight: np.ndarray | None = None,
          eps: float = 1e-6) -> np.ndarray:
    """Sum of rows 16 b + c_b of `table` (converted exactly to float64) per frame, then the
    optional RMSNorm with weight `rms_weight`; float64 [n_frames, dim]."""
    c = np.ascontiguousarray(codes_, np.uint8)
    assert c.ndim == 2 and c.shape[1] == NMEL
    T = np.ascontiguousarray(table, np.float64)
    assert T.shape[0] == NMEL * NLEV
    dim = T.shape[1]
    g = None if rms_weight is None else np.ascontiguousarray(rms_weight, np.float64)
    out = np.zeros((c.shape[0], dim), np.float64)
    rc = lib().oracle_embed(_ptr(c), c.shape[0], _ptr(T), dim, _ptr(g), float(eps), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_embed: code out of range")
    return out


# quantiser variants (modes of the C oracle): 0 uniform floor, 1 nearest of 16 reconstruction
# points, 2 mu-law companding; clamp range [lmin, lmax]
DEFAULT_QUANT = (LMIN, LMAX, 0, 0.0)


def log_clamp_q(M: float, lmin: float, lmax: float) -> float:
    return float(lib().oracle_log_clamp_q(float(M), float(lmin), float(lmax)))


def quantise_q(lhat: float, lmin: float, lmax: float, mode: int, mu: float = 0.0) -> int:
    return int(lib().oracle_quantise_q(float(lhat), float(lmin), float(lmax), int(mode), float(mu)))


def codes_q(wav: np.ndarray, sample_offsets: np.ndarray, quant, tails: np.ndarray | None = None,
            frame_ids: np.ndarray | None = None):
    """codes() under a quantiser variant quant = (lmin, lmax, mode, mu); returns (codes, lhat)
    with lhat clamped to [lmin, lmax]."""
    lmin, lmax, mode, mu = quant
    w = np.ascontiguousarray(wav, np.float32)
    so = np.ascontiguousarray(sample_offsets, np.int64)
    n_clips = so.shape[0] - 1
    t = None if tails is None else np.ascontiguousarray(tails, np.float32)
    if frame_ids is None:
        n = int(frame_offsets(so)[-1])
        ids = None
    else:
        ids = np.ascontiguousarray(frame_ids, np.int64)
        n = ids.shape[0]
    c = np.zeros((n, NMEL), np.uint8)
    lh = np.zeros((n, NMEL), np.float64)
    rc = lib().oracle_codes_q(_ptr(w), _ptr(so), n_clips, _ptr(t), _ptr(ids), n, float(lmin), float(lmax),
                              int(mode), float(mu), _ptr(c), _ptr(lh))
    if rc != 0:
        raise ValueError("oracle_codes_q: bad offsets or frame index")
    return c, lh


def level_boundaries_q(lmin: float, lmax: float, mode: int, mu: float = 0.0) -> np.ndarray:
    """The 15 inner decision boundaries in log-mel units of a quantiser variant (closed forms of
    the three mappings)."""
    k = np.arange(1, NLEV, dtype=np.float64)
    r = lmax - lmin
    if mode == 1:
        return lmin + r * (k - 0.5) / (NLEV - 1)
    if mode == 2:
        return lmin + r * (np.power(1.0 + mu, k / NLEV) - 1.0) / mu
    return lmin + r * k / NLEV


def boundary_distance_q(lhat: np.ndarray, quant) -> np.ndarray:
    bnd = level_boundaries_q(*quant)
    return np.min(np.abs(np.asarray(lhat)[..., None] - bnd), axis=-1)


def boundary_distance(lhat: np.ndarray) -> np.ndarray:
    """Distance of each clamped log-mel value to the nearest of the 15 inner level boundaries
    -7 + 9k/16, k = 1..15 (used by the agreement rule for codes)."""
    k = np.arange(1, NLEV, dtype=np.float64)
    bnd = LMIN + (LMAX - LMIN) * k / NLEV
    return np.min(np.abs(lhat[..., None] - bnd), axis=-1)


def splice(tokens: list, sentinel, frames_per_item: list) -> list:
    """Sentinel expansion ("Inside Inkling: Audio Design", Part 3 · Inference): at serve time an
    audio item is one sentinel token that expands into f frame positions. Written out plainly:
    walk the token list and replace the i-th sentinel by f_i entries ("frame", i, j); every other
    token is copied as ("token", original position). Returns the expanded list; its length and
    the positions of its entries are the splice plan. A clip with no frame leaves no entry."""
    out = []
    item = 0
    for pos, tok in enumerate(tokens):
        if tok == sentinel:
            for j in range(frames_per_item[item]):
                out.append(("frame", item, j))
            item += 1
        else:
            out.append(("token", pos))
    if item != len(frames_per_item):
        raise ValueError("one sentinel per audio item")
    return out


def splice_plan(seq_len: int, sentinel_pos: list, frames_per_item: list):
    """The splice plan read off the plain expansion: (token_pos [seq_len] with -1 at sentinels,
    frame_rows in frame order, expanded_len, audio_tokens)."""
    sentinel = object()
    tokens = [sentinel if p in set(sentinel_pos) else p for p in range(seq_len)]
    expanded = splice(tokens, sentinel, frames_per_item)
    token_pos = [-1] * seq_len
    frame_rows = [None] * sum(frames_per_item)
    starts = np.concatenate([[0], np.cumsum(frames_per_item)]).astype(int)
    for row, entry in enumerate(expanded):
        if entry[0] == "token":
            token_pos[entry[1]] = row
        else:
            frame_rows[starts[entry[1]] + entry[2]] = row
    return token_pos, frame_rows, len(expanded), int(sum(frames_per_item))


def shortconv(x: np.ndarray, seq_offsets, w: np.ndarray, state: np.ndarray | None = None):
    """ShortConv of tokens x [T, C] split into sequences by seq_offsets [n + 1], weights
    w [C, 4], carried states [n, 3, C] or None (zeros). Returns (y [T, C], state_out [n, 3, C]),
    all fp64 ("Inside Inkling: Audio Design", Part 3 · Inference: y = x + sum_d w_d x_{t-d})."""
    xx = np.ascontiguousarray(x, np.float64)
    off = np.ascontiguousarray(seq_offsets, np.int64)
    n = off.shape[0] - 1
    C = xx.shape[1]
    ww = np.ascontiguousarray(w, np.float64)
    assert ww.shape == (C, 4)
    st = None if state is None else np.ascontiguousarray(state, np.float64)
    y = np.zeros_like(xx)
    so = np.zeros((n, 3, C), np.float64)
    rc = lib().oracle_shortconv(_ptr(xx), _ptr(off), n, C, _ptr(ww), _ptr(st), _ptr(y), _ptr(so))
    if rc != 0:
        raise ValueError("oracle_shortconv: bad offsets")
    return y, so


# ---------------------------------------------------------------- hMLP patchifier (vision)

HMLP_PATCH = 40
HMLP_LN_EPS = 1e-6


def _bf16(a: np.ndarray) -> np.ndarray:
    """Round to bfloat16 (nearest even) and back to float64: the activations' storage type."""
    a32 = np.ascontiguousarray(a, np.float32)
    u = a32.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def _gelu(x: np.ndarray) -> np.ndarray:
    from math import erf, sqrt
    v = np.vectorize(lambda t: 0.5 * t * (1.0 + erf(t / sqrt(2.0))))
    return v(x) if x.size else x


def _layernorm(x: np.ndarray, g: np.ndarray, b: np.ndarray) -> np.ndarray:
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + HMLP_LN_EPS) * g + b


def hmlp(images: np.ndarray, params: dict) -> np.ndarray:
    """The hierarchical MLP patchifier ("Inside Inkling: Audio Design", Part 1 · Modeling: a
    4-layer hMLP over 40x40 patches; "Why Thinking Machines Built Inkling Without a Vision
    Encoder": linear layers progressively merge pixels into one embedding per patch), in fp64:
      stage 1: every 5x5 pixel block, its 75 values in (row, column, channel) order, times W1 + b1
      stages 2-4: every 2x2 group of the previous stage's grid, the four vectors concatenated in
               (top-left, top-right, bottom-left, bottom-right) order, times Ws + bs
    LayerNorm (eps 1e-6, gamma, beta) and the exact GELU follow stages 1-3; every stage's output
    is stored in bf16 (the input to the next stage and the final embedding). images: [n, H, W, 3]
    with H, W multiples of 40; returns [n * (H / 40) * (W / 40), D] with patches in raster order."""
    n, H, W, ch = images.shape
    assert ch == 3 and H % HMLP_PATCH == 0 and W % HMLP_PATCH == 0
    out = []
    for i in range(n):
        for pr in range(H // HMLP_PATCH):
            for pc in range(W // HMLP_PATCH):
                patch = np.asarray(images[i, 40 * pr:40 * pr + 40, 40 * pc:40 * pc + 40, :], np.float64)
                # stage 1: 8 x 8 grid of 5 x 5 blocks
                grid = np.zeros((8, 8, params["W1"].shape[1]))
                for br in range(8):
                    for bc in range(8):
                        v = patch[5 * br:5 * br + 5, 5 * bc:5 * bc + 5, :].reshape(-1)
                        grid[br, bc] = v @ params["W1"] + params["b1"]
                grid = _bf16(_gelu(_layernorm(grid, params["g1"], params["be1"])))
                for s in (2, 3, 4):
                    m = grid.shape[0] // 2
                    nxt = np.zeros((m, m, params[f"W{s}"].shape[1]))
                    for r in range(m):
                        for c in range(m):
                            v = np.concatenate([grid[2 * r, 2 * c], grid[2 * r, 2 * c + 1],
                                                grid[2 * r + 1, 2 * c], grid[2 * r + 1, 2 * c + 1]])
                            nxt[r, c] = v @ params[f"W{s}"] + params[f"b{s}"]
                    if s < 4:
                        nxt = _gelu(_layernorm(nxt, params[f"g{s}"], params[f"be{s}"]))
                    grid = _bf16(nxt)
                out.append(grid[0, 0])
    return np.stack(out) if out else np.zeros((0, params["W4"].shape[1]))
