"""Python binding of the dMel C ABI (include/dmel.h): argument marshalling only.

Every function here has the name of the C entry point it calls and passes device pointers of
torch tensors (plus the current CUDA stream) straight through; all computation runs in the
CUDA kernels of libdmel.so. The library must have been built (``encoder_free_audio_b200.build``);
importing this module without it raises, so nothing can silently fall back to another path.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_build", "libdmel.so")

DMEL_OK = 0
DMEL_ERR_INVALID_ARG = 1
DMEL_ERR_UNSUPPORTED = 2
DMEL_ERR_CUDA = 3
DMEL_ERR_TOO_LARGE = 4
DMEL_F32 = 0
DMEL_BF16 = 1
DMEL_DEVERR_CODE_RANGE = 0x1
DMEL_DEVERR_WAIT_TIMEOUT = 0x2
DMEL_DEVERR_OFFSETS = 0x4
DMEL_DEVERR_OUT_ROW = 0x8
DMEL_QUANT_FLOOR = 0
DMEL_QUANT_ROUND = 1
DMEL_QUANT_MULAW = 2


class Quantizer(ctypes.Structure):
    """dmel_quantizer: clamp range [min_value, max_value], mode (DMEL_QUANT_*), mu (mu-law)."""
    _fields_ = [("min_value", ctypes.c_float), ("max_value", ctypes.c_float), ("mode", ctypes.c_int),
                ("mu", ctypes.c_float)]

HOP = 800
WIN = 1600
N_MEL = 80
N_LEVELS = 16
TABLE_ROWS = 1280
MODEL_DIM = 6144


class DmelError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib().dmel_status_string(status).decode()}")


_L = None


def _lib():
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdmel.so is not built ({LIB_PATH}); run encoder_free_audio_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.dmel_frames_for_length.argtypes = [i64]
        L.dmel_frames_for_length.restype = i64
        L.dmel_frame_offsets.argtypes = [vp, i32, vp]
        L.dmel_frame_offsets.restype = i32
        L.dmel_workspace_size.argtypes = [i64, i32, i32, i32, i32]
        L.dmel_workspace_size.restype = sz
        L.dmel_codes.argtypes = [vp, vp, vp, i32, i64, vp, vp, vp, vp]
        L.dmel_codes.restype = i32
        L.dmel_embed.argtypes = [vp, i64, vp, i32, i32, vp, ctypes.c_float, vp, i32, vp, sz, vp]
        L.dmel_embed.restype = i32
        L.dmel_forward.argtypes = [vp, vp, vp, i32, i64, vp, vp, vp, i32, i32, vp, ctypes.c_float, vp, i32, vp, vp,
                                   sz, vp]
        L.dmel_forward.restype = i32
        L.dmel_table_prepare_size.argtypes = [i32, i32]
        L.dmel_table_prepare_size.restype = sz
        L.dmel_table_prepare.argtypes = [vp, i32, i32, vp, sz, vp]
        L.dmel_table_prepare.restype = i32
        L.dmel_embed_prepared.argtypes = [vp, i64, vp, i32, i32, vp, ctypes.c_float, vp, vp, i32, vp, sz, vp]
        L.dmel_embed_prepared.restype = i32
        L.dmel_forward_prepared.argtypes = [vp, vp, vp, i32, i64, vp, vp, vp, i32, i32, vp, ctypes.c_float, vp, vp,
                                            i32, vp, vp, sz, vp]
        L.dmel_forward_prepared.restype = i32
        L.dmel_embed_rows.argtypes = [vp, i64, vp, i32, i32, vp, ctypes.c_float, vp, vp, i64, i32, vp, sz, vp]
        L.dmel_embed_rows.restype = i32
        L.dmel_forward_rows.argtypes = [vp, vp, vp, i32, i64, vp, vp, vp, i32, i32, vp, ctypes.c_float, vp, vp, i64,
                                        i32, vp, vp, sz, vp]
        L.dmel_forward_rows.restype = i32
        L.dmel_splice_plan.argtypes = [vp, i32, vp, i64, vp, vp, ctypes.POINTER(i64), ctypes.POINTER(i64)]
        L.dmel_splice_plan.restype = i32
        L.dmel_hmlp_workspace_size.argtypes = [i64, ctypes.POINTER(HmlpWeights)]
        L.dmel_hmlp_workspace_size.restype = sz
        L.dmel_hmlp.argtypes = [vp, i32, i32, i32, ctypes.POINTER(HmlpWeights), vp, vp, sz, vp]
        L.dmel_hmlp.restype = i32
        L.dmel_shortconv.argtypes = [vp, vp, i32, i64, i32, vp, vp, vp, vp, i32, vp]
        L.dmel_shortconv.restype = i32
        L.dmel_embed_noalloc.argtypes = [vp, i64, vp, i32, i32, vp, ctypes.c_float, vp, i32, vp]
        L.dmel_embed_noalloc.restype = i32
        L.dmel_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
        L.dmel_get_device_error.restype = i32
        L.dmel_status_string.argtypes = [i32]
        L.dmel_status_string.restype = ctypes.c_char_p
        L.dmel_last_launch_count.argtypes = []
        L.dmel_last_launch_count.restype = i32
        L.dmel_debug_wait_timeout.argtypes = [ctypes.c_uint32, ctypes.POINTER(ctypes.c_uint32)]
        L.dmel_debug_wait_timeout.restype = i32
        L.dmel_debug_gelu.argtypes = [vp, vp, ctypes.c_int64, vp]
        L.dmel_debug_gelu.restype = i32
        L.dmel_debug_codes_frame_host.argtypes = [vp, vp, vp]
        L.dmel_debug_codes_frame_host.restype = None
        L.dmel_debug_codes_frame_host_q.argtypes = [vp, ctypes.POINTER(Quantizer), vp, vp]
        L.dmel_debug_codes_frame_host_q.restype = i32
        L.dmel_codes_q.argtypes = [vp, vp, vp, i32, i64, vp, vp, vp, ctypes.POINTER(Quantizer), vp]
        L.dmel_codes_q.restype = i32
        L.dmel_forward_host_workspace_size.argtypes = [vp, i32, i32, i32, i32, i32, i64]
        L.dmel_forward_host_workspace_size.restype = sz
        L.dmel_forward_host.argtypes = [vp, vp, i32, vp, i32, i32, vp, ctypes.c_float, vp, i32, vp, i64, vp, sz, vp]
        L.dmel_forward_host.restype = i32
        L.dmel_debug_forward_host_plan.argtypes = [vp, i32, i64, vp, i64, ctypes.POINTER(i64)]
        L.dmel_debug_forward_host_plan.restype = i32
        L.dmel_debug_gram.argtypes = [vp, i32, vp, vp]
        L.dmel_debug_gram.restype = i32
        L.dmel_debug_norm_sumsq_host.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_double)]
        L.dmel_debug_norm_sumsq_host.restype = i32
        L.dmel_debug_gemm.argtypes = [vp, i64, i32, i32, vp, i32, vp, vp]
        L.dmel_debug_gemm.restype = i32
        _L = L
    return _L


def library():
    """The loaded ctypes library (for symbol checks)."""
    return _lib()


# ---------------------------------------------------------------------------------- helpers

def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return DMEL_F32
    if t.dtype == torch.bfloat16:
        return DMEL_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check(rc: int, where: str):
    if rc != DMEL_OK:
        raise DmelError(rc, where)


# ---------------------------------------------------------------------------------- entry points

def dmel_frames_for_length(n_samples: int) -> int:
    return int(_lib().dmel_frames_for_length(int(n_samples)))


def dmel_frame_offsets(sample_offsets) -> np.ndarray:
    """Host int64 frame offsets [n_clips + 1] of host sample offsets."""
    so = np.ascontiguousarray(np.asarray(sample_offsets, dtype=np.int64))
    fo = np.zeros_like(so)
    rc = _lib().dmel_frame_offsets(so.ctypes.data_as(ctypes.c_void_p), so.shape[0] - 1,
                                   fo.ctypes.data_as(ctypes.c_void_p))
    _check(rc, "dmel_frame_offsets")
    return fo


def dmel_workspace_size(n_frames: int, embed_dim: int, table_dtype: int, with_rmsnorm: bool,
                        with_codes_out: bool) -> int:
    return int(_lib().dmel_workspace_size(int(n_frames), int(embed_dim), int(table_dtype), int(bool(with_rmsnorm)),
                                          int(bool(with_codes_out))))


def dmel_codes(wav, sample_offsets, frame_offsets, n_frames: int, codes, tails=None, tails_out=None, stream=None):
    """dmel_codes on torch CUDA tensors: wav fp32, offsets int64 [n_clips + 1], codes uint8
    [n_frames, 80], tails / tails_out fp32 [n_clips, 800] or None."""
    n_clips = sample_offsets.shape[0] - 1
    rc = _lib().dmel_codes(_ptr(wav), _ptr(sample_offsets), _ptr(frame_offsets), n_clips, int(n_frames), _ptr(tails),
                           _ptr(tails_out), _ptr(codes), _stream(stream))
    _check(rc, "dmel_codes")


def dmel_forward_host_workspace_size(sample_offsets, embed_dim: int, table_dtype: int, out_dtype: int,
                                     with_rmsnorm: bool, chunk_frames: int = 0) -> int:
    """Device workspace bytes of dmel_forward_host for these host sample offsets."""
    so = np.ascontiguousarray(np.asarray(sample_offsets, dtype=np.int64))
    return int(_lib().dmel_forward_host_workspace_size(so.ctypes.data_as(ctypes.c_void_p), so.shape[0] - 1,
                                                       int(embed_dim), int(table_dtype), int(out_dtype),
                                                       int(bool(with_rmsnorm)), int(chunk_frames)))


def dmel_forward_host(wav_host, sample_offsets, table, out_host, rms_weight=None, eps: float = 1e-6, codes_host=None,
                      chunk_frames: int = 0, workspace=None, stream=None):
    """dmel_forward_host: wav_host a host (pinned) fp32 torch tensor, sample_offsets host int64
    (numpy or list), table / rms_weight / workspace torch CUDA tensors, out_host a host tensor
    [F, D] (bf16 or fp32), codes_host None or host uint8 [F, 80]. Asynchronous on the stream."""
    so = np.ascontiguousarray(np.asarray(sample_offsets, dtype=np.int64))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib().dmel_forward_host(ctypes.c_void_p(wav_host.data_ptr()), so.ctypes.data_as(ctypes.c_void_p),
                                  so.shape[0] - 1, _ptr(table), _dtype_code(table), int(table.shape[1]),
                                  _ptr(rms_weight), ctypes.c_float(eps), ctypes.c_void_p(out_host.data_ptr()),
                                  _dtype_code(out_host), _ptr(codes_host), int(chunk_frames), _ptr(workspace),
                                  ws_bytes, _stream(stream))
    _check(rc, "dmel_forward_host")


class HmlpWeights(ctypes.Structure):
    """dmel_hmlp_weights: widths and device pointers of the hMLP patchifier's parameters."""
    _fields_ = [("d1", ctypes.c_int), ("d2", ctypes.c_int), ("d3", ctypes.c_int), ("dim", ctypes.c_int)] + \
               [(k, ctypes.c_void_p) for k in ("w1", "w2", "w3", "w4", "b1", "b2", "b3", "b4", "g1", "g2", "g3",
                                              "be1", "be2", "be3")]


def hmlp_weights(params: dict) -> HmlpWeights:
    """HmlpWeights of torch CUDA tensors: W1..W4 bf16 [75 x d1], [4 d1 x d2], [4 d2 x d3],
    [4 d3 x dim]; b1..b4, g1..g3, be1..be3 fp32."""
    d = [int(params[f"W{s}"].shape[1]) for s in (1, 2, 3, 4)]
    return HmlpWeights(*d, *[_ptr(params[k]) for k in ("W1", "W2", "W3", "W4", "b1", "b2", "b3", "b4", "g1", "g2",
                                                          "g3", "be1", "be2", "be3")])


def dmel_hmlp_workspace_size(n_patches: int, params: dict) -> int:
    return int(_lib().dmel_hmlp_workspace_size(int(n_patches), ctypes.byref(hmlp_weights(params))))


def dmel_hmlp(images, params: dict, out, workspace, stream=None):
    """dmel_hmlp on torch CUDA tensors: images bf16 [n, H, W, 3], out bf16 [patches, dim]."""
    n, H, W, _ = images.shape
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = _lib().dmel_hmlp(_ptr(images), int(n), int(H), int(W), ctypes.byref(hmlp_weights(params)), _ptr(out),
                          _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "dmel_hmlp")


def _quantizer(q):
    """None, a Quantizer, or a tuple (min_value, max_value, mode, mu)."""
    if q is None or isinstance(q, Quantizer):
        return q
    lo, hi, mode, mu = q
    return Quantizer(float(lo), float(hi), int(mode), float(mu))


def dmel_codes_q(wav, sample_offsets, frame_offsets, n_frames: int, codes, quantizer=None, tails=None, tails_out=None,
                 stream=None):
    """dmel_codes_q on torch CUDA tensors: dmel_codes with the level mapping `quantizer`
    (None, a Quantizer, or (min_value, max_value, mode, mu))."""
    n_clips = sample_offsets.shape[0] - 1
    q = _quantizer(quantizer)
    rc = _lib().dmel_codes_q(_ptr(wav), _ptr(sample_offsets), _ptr(frame_offsets), n_clips, int(n_frames), _ptr(tails),
                             _ptr(tails_out), _ptr(codes), None if q is None else ctypes.byref(q), _stream(stream))
    _check(rc, "dmel_codes_q")


def dmel_embed(codes, table, out, rms_weight=None, eps: float = 1e-6, workspace=None, stream=None):
    """dmel_embed on torch CUDA tensors: codes uint8 [F, 80], table [1280, D] fp32/bf16,
    out [F, D] fp32/bf16, rms_weight [D] in the table's dtype or None, workspace uint8 or None."""
    n = codes.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib().dmel_embed(_ptr(codes), n, _ptr(table), _dtype_code(table), table.shape[1], _ptr(rms_weight),
                           float(eps), _ptr(out), _dtype_code(out), _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "dmel_embed")


def dmel_embed_noalloc(codes, table, out, rms_weight=None, eps: float = 1e-6, stream=None):
    """dmel_embed_noalloc on torch CUDA tensors: dmel_embed without a workspace, for callers
    that cannot allocate (the library's fixed 4 MiB scratch is used instead)."""
    n = codes.shape[0]
    rc = _lib().dmel_embed_noalloc(_ptr(codes), n, _ptr(table), _dtype_code(table), table.shape[1],
                                   _ptr(rms_weight), float(eps), _ptr(out), _dtype_code(out), _stream(stream))
    _check(rc, "dmel_embed_noalloc")


def dmel_forward(wav, sample_offsets, frame_offsets, n_frames: int, table, out, rms_weight=None, eps: float = 1e-6,
                 tails=None, tails_out=None, codes_out=None, workspace=None, stream=None):
    """dmel_forward on torch CUDA tensors (see dmel_codes and dmel_embed for the arguments)."""
    n_clips = sample_offsets.shape[0] - 1
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib().dmel_forward(_ptr(wav), _ptr(sample_offsets), _ptr(frame_offsets), n_clips, int(n_frames),
                             _ptr(tails), _ptr(tails_out), _ptr(table), _dtype_code(table), table.shape[1],
                             _ptr(rms_weight), float(eps), _ptr(out), _dtype_code(out), _ptr(codes_out),
                             _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "dmel_forward")


def dmel_table_prepare_size(embed_dim: int, table_dtype: int) -> int:
    """Bytes of a table's prepared data (its Gram matrix), 0 when none applies."""
    return int(_lib().dmel_table_prepare_size(int(embed_dim), int(table_dtype)))


def dmel_table_prepare(table, prepared, stream=None):
    """G = T T^T of a bf16 CUDA table [1280, D] into the CUDA uint8 tensor prepared (at least
    dmel_table_prepare_size bytes)."""
    rc = _lib().dmel_table_prepare(_ptr(table), table.shape[1], _dtype_code(table), _ptr(prepared),
                                   prepared.numel() * prepared.element_size(), _stream(stream))
    _check(rc, "dmel_table_prepare")


def dmel_embed_prepared(codes, table, out, prepared, rms_weight=None, eps: float = 1e-6, workspace=None, stream=None):
    """dmel_embed with the table's prepared data (or None)."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib().dmel_embed_prepared(_ptr(codes), int(codes.shape[0]), _ptr(table), _dtype_code(table), table.shape[1],
                                    _ptr(rms_weight), float(eps), _ptr(prepared), _ptr(out), _dtype_code(out),
                                    _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "dmel_embed_prepared")


def dmel_forward_prepared(wav, sample_offsets, frame_offsets, n_frames: int, table, out, prepared, rms_weight=None,
                          eps: float = 1e-6, tails=None, tails_out=None, codes_out=None, workspace=None, stream=None):
    """dmel_forward with the table's prepared data (or None)."""
    n_clips = sample_offsets.shape[0] - 1
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib().dmel_forward_prepared(_ptr(wav), _ptr(sample_offsets), _ptr(frame_offsets), n_clips, int(n_frames),
                                      _ptr(tails), _ptr(tails_out), _ptr(table), _dtype_code(table), table.shape[1],
                                      _ptr(rms_weight), float(eps), _ptr(prepared), _ptr(out), _dtype_code(out),
                                      _ptr(codes_out), _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "dmel_forward_prepared")


def dmel_embed_rows(codes, table, out, out_rows, rms_weight=None, eps: float = 1e-6, workspace=None, stream=None):
    """dmel_embed_rows on torch CUDA tensors: as dmel_embed, frame f written to row out_rows[f]
    (int64 [F] on the device) of out [S, D]."""
    n = codes.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib().dmel_embed_rows(_ptr(codes), n, _ptr(table), _dtype_code(table), table.shape[1], _ptr(rms_weight),
                                float(eps), _ptr(out), _ptr(out_rows), int(out.shape[0]), _dtype_code(out),
                                _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "dmel_embed_rows")


def dmel_forward_rows(wav, sample_offsets, frame_offsets, n_frames: int, table, out, out_rows, rms_weight=None,
                      eps: float = 1e-6, tails=None, tails_out=None, codes_out=None, workspace=None, stream=None):
    """dmel_forward_rows on torch CUDA tensors: as dmel_forward, frame f written to row
    out_rows[f] (int64 [n_frames] on the device) of out [S, D]."""
    n_clips = sample_offsets.shape[0] - 1
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib().dmel_forward_rows(_ptr(wav), _ptr(sample_offsets), _ptr(frame_offsets), n_clips, int(n_frames),
                                  _ptr(tails), _ptr(tails_out), _ptr(table), _dtype_code(table), table.shape[1],
                                  _ptr(rms_weight), float(eps), _ptr(out), _ptr(out_rows), int(out.shape[0]),
                                  _dtype_code(out), _ptr(codes_out), _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "dmel_forward_rows")


def dmel_shortconv(x, seq_offsets, weights, y, state=None, state_out=None, stream=None):
    """dmel_shortconv on torch CUDA tensors: x and y [T, C] (fp32 or bf16), seq_offsets int64
    [n + 1], weights fp32 [C, 4], state / state_out [n, 3, C] in x's dtype or None."""
    n_seq = seq_offsets.shape[0] - 1
    rc = _lib().dmel_shortconv(_ptr(x), _ptr(seq_offsets), n_seq, int(x.shape[0]), int(x.shape[1]), _ptr(weights),
                               _ptr(state), _ptr(state_out), _ptr(y), _dtype_code(x), _stream(stream))
    _check(rc, "dmel_shortconv")


def dmel_splice_plan(sentinel_pos, frame_offsets, seq_len: int):
    """Host splice plan: (token_pos [seq_len], frame_rows [F], expanded_len, audio_tokens) for a
    sequence of seq_len positions with audio sentinels at sentinel_pos (one per clip of
    frame_offsets)."""
    sp = np.ascontiguousarray(np.asarray(sentinel_pos, dtype=np.int64))
    fo = np.ascontiguousarray(np.asarray(frame_offsets, dtype=np.int64))
    n_items = sp.shape[0]
    if fo.shape[0] != n_items + 1:
        raise DmelError(DMEL_ERR_INVALID_ARG, "dmel_splice_plan (frame offsets must have n_items + 1 entries)")
    token_pos = np.empty(max(int(seq_len), 0), dtype=np.int64)
    frame_rows = np.empty(int(fo[-1]) if fo.shape[0] else 0, dtype=np.int64)
    exp_len, audio = ctypes.c_int64(0), ctypes.c_int64(0)
    rc = _lib().dmel_splice_plan(sp.ctypes.data_as(ctypes.c_void_p), n_items, fo.ctypes.data_as(ctypes.c_void_p),
                                 int(seq_len), token_pos.ctypes.data_as(ctypes.c_void_p),
                                 frame_rows.ctypes.data_as(ctypes.c_void_p), ctypes.byref(exp_len),
                                 ctypes.byref(audio))
    _check(rc, "dmel_splice_plan")
    return token_pos, frame_rows, int(exp_len.value), int(audio.value)


def dmel_get_device_error(clear: bool = True) -> int:
    bits = ctypes.c_uint32(0)
    rc = _lib().dmel_get_device_error(ctypes.byref(bits), int(clear))
    _check(rc, "dmel_get_device_error")
    return int(bits.value)


def dmel_status_string(status: int) -> str:
    return _lib().dmel_status_string(int(status)).decode()


def dmel_last_launch_count() -> int:
    return int(_lib().dmel_last_launch_count())


def dmel_debug_codes_frame_host(frame1600: np.ndarray):
    """Host emulation of the codes kernel's per-frame arithmetic (diagnostic, see dmel_debug.h)."""
    fr = np.ascontiguousarray(frame1600, np.float32)
    assert fr.shape == (WIN,)
    codes = np.zeros(N_MEL, np.uint8)
    lhat = np.zeros(N_MEL, np.float64)
    _lib().dmel_debug_codes_frame_host(fr.ctypes.data_as(ctypes.c_void_p), codes.ctypes.data_as(ctypes.c_void_p),
                                       lhat.ctypes.data_as(ctypes.c_void_p))
    return codes, lhat


def dmel_debug_codes_frame_host_q(frame1600: np.ndarray, quantizer=None):
    """Host emulation with the level mapping `quantizer` (as dmel_codes_q)."""
    fr = np.ascontiguousarray(frame1600, np.float32)
    assert fr.shape == (WIN,)
    codes = np.zeros(N_MEL, np.uint8)
    lhat = np.zeros(N_MEL, np.float64)
    q = _quantizer(quantizer)
    rc = _lib().dmel_debug_codes_frame_host_q(fr.ctypes.data_as(ctypes.c_void_p), None if q is None else ctypes.byref(q),
                                              codes.ctypes.data_as(ctypes.c_void_p),
                                              lhat.ctypes.data_as(ctypes.c_void_p))
    _check(rc, "dmel_debug_codes_frame_host_q")
    return codes, lhat


def dmel_debug_gelu(x, y=None):
    """GELU of a contiguous fp32 device tensor with the hMLP kernels' formula (diagnostic, see
    dmel_debug.h); returns y."""
    import torch
    if y is None:
        y = torch.empty_like(x)
    rc = _lib().dmel_debug_gelu(_ptr(x), _ptr(y), x.numel(), _stream(None))
    _check(rc, "dmel_debug_gelu")
    return y


def dmel_debug_wait_timeout(polls: int = 1 << 16) -> int:
    """Runs the bounded-wait self test (see dmel_debug.h); returns the device error bits."""
    bits = ctypes.c_uint32(0)
    rc = _lib().dmel_debug_wait_timeout(int(polls), ctypes.byref(bits))
    _check(rc, "dmel_debug_wait_timeout")
    return int(bits.value)


def dmel_debug_forward_host_plan(sample_offsets, chunk_frames: int) -> list:
    """dmel_forward_host's chunk plan (diagnostic, see dmel_debug.h) as a list of dicts with keys
    f0, f1, s_lo, s_hi, tail, so, fo."""
    so = np.ascontiguousarray(np.asarray(sample_offsets, dtype=np.int64))
    n = ctypes.c_int64(0)
    _check(_lib().dmel_debug_forward_host_plan(so.ctypes.data_as(ctypes.c_void_p), so.shape[0] - 1,
                                               int(chunk_frames), None, 0, ctypes.byref(n)),
           "dmel_debug_forward_host_plan")
    buf = np.zeros(max(1, n.value), np.int64)
    _check(_lib().dmel_debug_forward_host_plan(so.ctypes.data_as(ctypes.c_void_p), so.shape[0] - 1,
                                               int(chunk_frames), buf.ctypes.data_as(ctypes.c_void_p), n.value,
                                               ctypes.byref(n)), "dmel_debug_forward_host_plan")
    out, i = [], 0
    while i < n.value:
        f0, f1, s_lo, s_hi, tail, k = (int(v) for v in buf[i:i + 6])
        i += 6
        out.append({"f0": f0, "f1": f1, "s_lo": s_lo, "s_hi": s_hi, "tail": bool(tail),
                    "so": buf[i:i + k + 1].copy(), "fo": buf[i + k + 1:i + 2 * k + 2].copy()})
        i += 2 * k + 2
    return out


def dmel_debug_gram(table, gram, stream=None):
    """G = T T^T of a bf16 CUDA table [1280, D] into gram[0] of the CUDA fp32 tensor gram
    [2, 1280, 1280] (the upper blocks; gram[1] is scratch; diagnostic, see dmel_debug.h)."""
    assert gram.shape == (2, 1280, 1280)
    _check(_lib().dmel_debug_gram(_ptr(table), int(table.shape[1]), _ptr(gram), _stream(stream)), "dmel_debug_gram")


def dmel_debug_gemm(a, b, c, stream=None):
    """c [m, n] fp32 = a [m, k] bf16 @ b [k, n] bf16 on the hMLP stage GEMM (CUDA tensors; a may
    be a row slice of a wider array: its row stride is passed; diagnostic, see dmel_debug.h)."""
    m, k = a.shape
    assert b.shape[0] == k and c.shape == (m, b.shape[1]) and b.is_contiguous() and c.is_contiguous()
    assert a.stride(1) == 1
    _check(_lib().dmel_debug_gemm(_ptr(a), int(m), int(k), int(a.stride(0)), _ptr(b), int(b.shape[1]), _ptr(c),
                                  _stream(stream)), "dmel_debug_gemm")


def dmel_debug_norm_sumsq_host(codes80: np.ndarray, gram: np.ndarray) -> float:
    """The device's per-frame sum of squares from G, evaluated on the host (diagnostic)."""
    c = np.ascontiguousarray(codes80, np.uint8)
    g = np.ascontiguousarray(gram, np.float32)
    out = ctypes.c_double(0.0)
    _check(_lib().dmel_debug_norm_sumsq_host(c.ctypes.data_as(ctypes.c_void_p), g.ctypes.data_as(ctypes.c_void_p),
                                             ctypes.byref(out)), "dmel_debug_norm_sumsq_host")
    return out.value
