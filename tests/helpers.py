"""Comparison helpers shared by the GPU parity tests (agreement rules of the front end:
codes equal except within 1e-4 of a level boundary; embeddings within rtol of
max(|o_j|, rms of the oracle row))."""
import numpy as np


def compare_codes(gpu_codes: np.ndarray, ora_codes: np.ndarray, ora_lhat: np.ndarray, band: float = 1e-4,
                  boundaries: np.ndarray | None = None):
    """Returns (number of flipped cells, boolean mask of frames with a flip). Fails on any
    mismatch whose oracle value lies farther than `band` from every inner level boundary
    (the default mapping's, -7 + 9k/16, unless `boundaries` gives a variant's)."""
    assert gpu_codes.shape == ora_codes.shape, (gpu_codes.shape, ora_codes.shape)
    if boundaries is None:
        k = np.arange(1, 16, dtype=np.float64)
        bnd = -7.0 + 9.0 * k / 16.0
    else:
        bnd = np.asarray(boundaries, np.float64)
    mism = gpu_codes != ora_codes
    if not mism.any():
        return 0, np.zeros(gpu_codes.shape[0], bool)
    idx = np.nonzero(mism)
    dist = np.min(np.abs(ora_lhat[idx][:, None] - bnd[None, :]), axis=1)
    bad = dist > band
    assert not bad.any(), (f"{int(bad.sum())} code mismatches away from a level boundary, first at "
                           f"frame {idx[0][bad][0]} channel {idx[1][bad][0]}: gpu {gpu_codes[idx][bad][0]} "
                           f"oracle {ora_codes[idx][bad][0]} L {ora_lhat[idx][bad][0]}")
    step = np.abs(gpu_codes[idx].astype(int) - ora_codes[idx].astype(int))
    assert (step == 1).all(), "a flip near a boundary must be to the neighbouring level"
    return int(mism.sum()), mism.any(axis=1)


def compare_embed(gpu: np.ndarray, ora: np.ndarray, rtol: float):
    """Elementwise |y - o| <= rtol * max(|o_j|, rms(o_row)); returns the worst ratio
    |y - o| / max(|o_j|, rms(o_row)) so tests can report it."""
    g = np.asarray(gpu, np.float64)
    assert g.shape == ora.shape, (g.shape, ora.shape)
    rms = np.sqrt(np.mean(ora * ora, axis=1, keepdims=True))
    scale = np.maximum(np.abs(ora), rms)
    scale = np.where(scale > 0, scale, 1e-30)
    ratio = np.abs(g - ora) / scale
    worst = float(ratio.max()) if ratio.size else 0.0
    assert np.isfinite(g).all(), "non-finite output"
    assert worst <= rtol, f"embedding error {worst:.3e} > {rtol:.1e}"
    return worst


def bf16_table(table_f32: np.ndarray):
    """(torch bf16 tensor on CPU, exact float64 copy of it)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(table_f32)).to(torch.bfloat16)
    return t, t.float().numpy().astype(np.float64)
