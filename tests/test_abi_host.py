"""CPU tests of the C ABI: the library loads, exports what the headers declare, and its host
logic (frame counts, offsets, workspace sizing, argument checks) behaves without a GPU.
Also checks the codes kernel's per-frame arithmetic, run lane by lane on the host through
dmel_debug_codes_frame_host, against the oracle."""
import ctypes
import os
import re

import numpy as np
import pytest

from encoder_free_audio_b200 import build, dmel, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return dmel.library()


def _declared(header):
    txt = open(os.path.join(ROOT, "include", header)).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(dmel_[a-z_0-9]+)\s*\(", txt)))


def test_exports_every_declared_symbol(lib):
    names = _declared("dmel.h") + _declared("dmel_debug.h")
    assert "dmel_forward" in names and "dmel_codes" in names and "dmel_embed" in names
    for n in names:
        assert hasattr(lib, n), n


def test_frame_counts(lib):
    assert [dmel.dmel_frames_for_length(n) for n in (0, 799, 800, 32000, 160000, 19_200_000)] == [0, 0, 1, 40, 200,
                                                                                                 24000]
    assert dmel.dmel_frames_for_length(-5) == -1


def test_frame_offsets_host(lib, oracle_mod):
    so = synth.offsets_from_lengths([800, 0, 2399, 799, 5000, 1600, 16000 * 30])
    np.testing.assert_array_equal(dmel.dmel_frame_offsets(so), oracle_mod.frame_offsets(so))
    with pytest.raises(dmel.DmelError):
        dmel.dmel_frame_offsets(np.array([0, 10, 5]))
    with pytest.raises(dmel.DmelError):
        dmel.dmel_frame_offsets(np.array([3, 10]))


def test_workspace_size(lib):
    F = 12800
    assert dmel.dmel_workspace_size(0, 6144, dmel.DMEL_BF16, True, False) == 0
    with_codes = dmel.dmel_workspace_size(F, 6144, dmel.DMEL_BF16, True, True)
    r256 = lambda x: (x + 255) // 256 * 256
    # the larger of: G [1280 x 1280] fp32 and its second partial product + 55 partial sums of
    # squares per frame + one scale per frame + the sparse product's tile counter (RMSNorm from
    # the Gram matrix, dynamic tile schedule); row sums of squares
    # [frame tiles of 128][column tiles of 192][128] fp32 + one counter per frame tile (the
    # exchange between a row's CTAs)
    gram = 2 * r256(1280 * 1280 * 4) + r256(55 * F * 4) + r256(F * 4) + 256
    tiles = (F + 127) // 128
    exchange = r256(tiles * 32 * 128 * 4) + r256(tiles * 4)
    assert with_codes == max(gram, exchange)
    assert dmel.dmel_workspace_size(F, 6144, dmel.DMEL_BF16, True, False) == with_codes + F * 80
    assert dmel.dmel_workspace_size(F, 6144, dmel.DMEL_BF16, False, True) == 0
    assert dmel.dmel_workspace_size(F, 6144, dmel.DMEL_F32, True, True) == 0  # CUDA-core path


def test_argument_checks_return_invalid_arg_without_gpu(lib):
    vp = ctypes.c_void_p
    fake = vp(1 << 20)  # never dereferenced: every call below fails its host checks first
    # negative sizes
    assert lib.dmel_codes(fake, fake, fake, -1, 0, None, None, fake, None) == dmel.DMEL_ERR_INVALID_ARG
    assert lib.dmel_codes(fake, fake, fake, 1, -1, None, None, fake, None) == dmel.DMEL_ERR_INVALID_ARG
    # frames without clips, missing offsets, missing codes
    assert lib.dmel_codes(fake, fake, fake, 0, 5, None, None, fake, None) == dmel.DMEL_ERR_INVALID_ARG
    assert lib.dmel_codes(fake, None, fake, 2, 5, None, None, fake, None) == dmel.DMEL_ERR_INVALID_ARG
    assert lib.dmel_codes(fake, fake, fake, 2, 5, None, None, None, None) == dmel.DMEL_ERR_INVALID_ARG
    # zero clips is a no-op
    assert lib.dmel_codes(None, None, None, 0, 0, None, None, None, None) == dmel.DMEL_OK
    E = lib.dmel_embed
    # embed_dim not a multiple of 8, bad dtype, missing pointers, misaligned output, eps <= 0
    assert E(fake, 4, fake, 1, 6100, None, 1e-6, fake, 1, None, 0, None) == dmel.DMEL_ERR_INVALID_ARG
    assert E(fake, 4, fake, 7, 6144, None, 1e-6, fake, 1, None, 0, None) == dmel.DMEL_ERR_INVALID_ARG
    assert E(None, 4, fake, 1, 6144, None, 1e-6, fake, 1, None, 0, None) == dmel.DMEL_ERR_INVALID_ARG
    assert E(fake, 4, None, 1, 6144, None, 1e-6, fake, 1, None, 0, None) == dmel.DMEL_ERR_INVALID_ARG
    assert E(fake, 4, fake, 1, 6144, None, 1e-6, vp((1 << 20) + 2), 1, None, 0, None) == dmel.DMEL_ERR_INVALID_ARG
    assert E(fake, 4, fake, 1, 6144, fake, 0.0, fake, 1, None, 0, None) == dmel.DMEL_ERR_INVALID_ARG
    # RMSNorm on the tensor-core path without the workspace it needs
    assert E(fake, 4, fake, 1, 6144, fake, 1e-6, fake, 1, None, 0, None) == dmel.DMEL_ERR_INVALID_ARG
    # CUDA-core path is limited to D <= 16384
    assert E(fake, 4, fake, 0, 16392, None, 1e-6, fake, 0, None, 0, None) == dmel.DMEL_ERR_INVALID_ARG
    # zero frames is a no-op
    assert E(None, 0, None, 1, 6144, None, 1e-6, None, 1, None, 0, None) == dmel.DMEL_OK
    # row-mapped output: a row map needs a positive row count and 8-byte alignment
    R = lib.dmel_embed_rows
    assert R(fake, 4, fake, 1, 6144, None, 1e-6, fake, fake, 0, 1, None, 0, None) == dmel.DMEL_ERR_INVALID_ARG
    assert R(fake, 4, fake, 1, 6144, None, 1e-6, fake, vp((1 << 20) + 4), 10, 1, None, 0,
             None) == dmel.DMEL_ERR_INVALID_ARG
    assert R(None, 0, None, 1, 6144, None, 1e-6, None, None, 0, 1, None, 0, None) == dmel.DMEL_OK
    FR = lib.dmel_forward_rows
    assert FR(fake, fake, fake, 1, 4, None, None, fake, 1, 6144, None, 1e-6, fake, fake, -3, 1, fake, None, 0,
              None) == dmel.DMEL_ERR_INVALID_ARG
    Fw = lib.dmel_forward
    assert Fw(fake, fake, fake, 1, 4, None, None, fake, 1, 6144, fake, 1e-6, fake, 1, None, None, 0,
              None) == dmel.DMEL_ERR_INVALID_ARG  # no workspace for codes + partial sums
    assert Fw(None, None, None, 0, 0, None, None, fake, 1, 6144, None, 1e-6, fake, 1, None, None, 0,
              None) == dmel.DMEL_OK
    bits = ctypes.c_uint32(0)
    assert lib.dmel_get_device_error(None, 0) == dmel.DMEL_ERR_INVALID_ARG
    del bits


def test_status_strings(lib):
    for s in range(4):
        assert dmel.dmel_status_string(s).startswith("DMEL_")
    assert dmel.dmel_status_string(99) == "DMEL_ERR_UNKNOWN"


def _frames(wav, off, ids, oracle_mod):
    """Raw 1600-sample frames of the listed global frames under the causal framing."""
    fo = oracle_mod.frame_offsets(off)
    out = np.zeros((len(ids), 1600), np.float32)
    for i, g in enumerate(ids):
        c = int(np.searchsorted(fo, g, side="right") - 1)
        t = g - fo[c]
        for n in range(1600):
            j = 800 * (t - 1) + n
            out[i, n] = wav[off[c] + j] if j >= 0 else 0.0
    return out


def _compare_codes(gc, gl, oc, ol, oracle_mod):
    dist = oracle_mod.boundary_distance(ol)
    mism = gc != oc
    assert not (mism & (dist > 1e-4)).any(), "code mismatch away from a level boundary"
    inner = (ol > -7.0) & (ol < 2.0)
    # the DFT runs in fp64, the mel sums and log10 in fp32: ~1e-7 in L
    np.testing.assert_allclose(gl[inner], ol[inner], rtol=0, atol=2e-6)


def test_kernel_arithmetic_on_host_matches_oracle(lib, oracle_mod):
    wav, off = synth.one_clip_2s()
    ids = np.arange(40)
    frames = _frames(wav, off, ids, oracle_mod)
    oc, ol = oracle_mod.codes(wav, off)
    for i in range(40):
        gc, gl = dmel.dmel_debug_codes_frame_host(frames[i])
        _compare_codes(gc, gl, oc[i], ol[i], oracle_mod)


def test_kernel_arithmetic_on_host_tones_and_noise(lib, oracle_mod):
    r = np.random.default_rng(11)
    n = np.arange(1600)
    cases = [np.zeros(1600), np.cos(2 * np.pi * 100 * n / 1600), 0.3 * np.cos(2 * np.pi * 3.37 * n / 1600 + 1.0),
             r.uniform(-1, 1, 1600), 1e-5 * r.standard_normal(1600),
             synth.harmonic_tone(1600, 123.4, 0.4, 10, 0.3)]
    for x in cases:
        fr = x.astype(np.float32)
        gc, gl = dmel.dmel_debug_codes_frame_host(fr)
        oc, ol = oracle_mod.codes(fr, np.array([0, 1600]), tails=None, frame_ids=np.array([1]))
        _compare_codes(gc, gl, oc[0], ol[0], oracle_mod)


def test_kernel_arithmetic_on_host_extremes(lib, oracle_mod):
    """Frames at the ends of the range: a NaN sample (every energy NaN: read as the floor, so
    code 0 everywhere), a constant 1e30 frame (the fp32 mel sums overflow, L clamps at the top),
    and a 1e-30 frame (the energies underflow, L clamps at the bottom): the same codes as the
    oracle, all in 0..15."""
    r = np.random.default_rng(12)
    nan_frame = r.uniform(-0.5, 0.5, 1600).astype(np.float32)
    nan_frame[777] = np.nan
    cases = [nan_frame, np.full(1600, 1e30, np.float32),
             (1e-30 * r.standard_normal(1600)).astype(np.float32)]
    for fr in cases:
        gc, _ = dmel.dmel_debug_codes_frame_host(fr)
        oc, _ = oracle_mod.codes(fr, np.array([0, 1600]), tails=None, frame_ids=np.array([1]))
        np.testing.assert_array_equal(gc, oc[0])
        assert gc.max() <= 15
    assert (dmel.dmel_debug_codes_frame_host(cases[0])[0] == 0).all()
    assert (dmel.dmel_debug_codes_frame_host(cases[1])[0] == 15).all()
    assert (dmel.dmel_debug_codes_frame_host(cases[2])[0] == 0).all()


# ---------------------------------------------------------------- quantiser variants on the host

QUANTS = [(-7.0, 2.0, dmel.DMEL_QUANT_FLOOR, 0.0), (-1.5, 2.0, dmel.DMEL_QUANT_FLOOR, 0.0),
          (-7.0, 2.0, dmel.DMEL_QUANT_ROUND, 0.0), (-1.5, 2.0, dmel.DMEL_QUANT_ROUND, 0.0),
          (-7.0, 2.0, dmel.DMEL_QUANT_MULAW, 255.0), (-1.5, 2.0, dmel.DMEL_QUANT_MULAW, 255.0)]


@pytest.mark.parametrize("q", QUANTS)
def test_kernel_quantiser_variants_on_host_match_oracle(lib, oracle_mod, q):
    wav, off = synth.one_clip_2s()
    frames = _frames(wav, off, np.arange(40), oracle_mod)
    oc, ol = oracle_mod.codes_q(wav, off, q)
    for i in range(40):
        gc, gl = dmel.dmel_debug_codes_frame_host_q(frames[i], q)
        dist = oracle_mod.boundary_distance_q(ol[i], q)
        assert not ((gc != oc[i]) & (dist > 1e-4)).any(), "code mismatch away from a level boundary"
        inner = (ol[i] > q[0]) & (ol[i] < q[1])
        np.testing.assert_allclose(gl[inner], ol[i][inner], rtol=0, atol=2e-6)


def test_default_quantiser_is_bit_identical_on_host(lib):
    wav, off = synth.one_clip_2s()
    r = np.random.default_rng(3)
    for t in range(1, 40, 7):
        fr = wav[800 * (t - 1):800 * (t + 1)].astype(np.float32)
        c0, l0 = dmel.dmel_debug_codes_frame_host(fr)
        c1, l1 = dmel.dmel_debug_codes_frame_host_q(fr, None)
        c2, l2 = dmel.dmel_debug_codes_frame_host_q(fr, (-7.0, 2.0, dmel.DMEL_QUANT_FLOOR, 0.0))
        assert (c0 == c1).all() and (c0 == c2).all() and (l0 == l1).all() and (l0 == l2).all()


@pytest.mark.parametrize("q", [(2.0, 2.0, 0, 0.0), (3.0, -7.0, 0, 0.0), (float("nan"), 2.0, 0, 0.0),
                               (-7.0, float("inf"), 0, 0.0), (-7.0, 2.0, 3, 0.0), (-7.0, 2.0, 2, 0.0),
                               (-7.0, 2.0, 2, -1.0)])
def test_bad_quantisers_are_rejected_without_gpu(lib, q):
    fr = np.zeros(1600, np.float32)
    with pytest.raises(dmel.DmelError):
        dmel.dmel_debug_codes_frame_host_q(fr, q)
    vp = ctypes.c_void_p
    fake = vp(1 << 20)
    qq = dmel.Quantizer(*q)
    assert lib.dmel_codes_q(fake, fake, fake, 1, 4, None, None, fake, ctypes.byref(qq),
                            None) == dmel.DMEL_ERR_INVALID_ARG


def test_shortconv_argument_checks_without_gpu(lib):
    vp = ctypes.c_void_p
    a, b, c = vp(1 << 20), vp(1 << 24), vp(1 << 28)
    S = lib.dmel_shortconv
    # channels not a multiple of 8, negative sizes, tokens without sequences
    assert S(a, a, 1, 10, 12, b, None, None, c, 1, None) == dmel.DMEL_ERR_INVALID_ARG
    assert S(a, a, -1, 10, 16, b, None, None, c, 1, None) == dmel.DMEL_ERR_INVALID_ARG
    assert S(a, a, 0, 10, 16, b, None, None, c, 1, None) == dmel.DMEL_ERR_INVALID_ARG
    # misaligned weights, missing output
    assert S(a, a, 1, 10, 16, vp((1 << 24) + 4), None, None, c, 1, None) == dmel.DMEL_ERR_INVALID_ARG
    assert S(a, a, 1, 10, 16, b, None, None, None, 1, None) == dmel.DMEL_ERR_INVALID_ARG
    # y overlapping x (in place is not allowed)
    assert S(a, a, 1, 10, 16, b, None, None, vp((1 << 20) + 64), 1, None) == dmel.DMEL_ERR_INVALID_ARG
    # no sequences: a no-op
    assert S(None, None, 0, 0, 16, None, None, None, None, 1, None) == dmel.DMEL_OK


def test_hmlp_argument_checks_without_gpu(lib):
    vp = ctypes.c_void_p
    a = vp(1 << 20)
    w = dmel.HmlpWeights(16, 16, 16, 32, *([a] * 14))
    H = lib.dmel_hmlp
    # height / width not multiples of 40
    assert H(a, 1, 40, 50, ctypes.byref(w), a, a, 1 << 30, None) == dmel.DMEL_ERR_INVALID_ARG
    # a width that is not a multiple of 8, a missing or misaligned parameter
    bad = dmel.HmlpWeights(16, 12, 16, 32, *([a] * 14))
    assert H(a, 1, 40, 40, ctypes.byref(bad), a, a, 1 << 30, None) == dmel.DMEL_ERR_INVALID_ARG
    miss = dmel.HmlpWeights(16, 16, 16, 32, *([a] * 13 + [None]))
    assert H(a, 1, 40, 40, ctypes.byref(miss), a, a, 1 << 30, None) == dmel.DMEL_ERR_INVALID_ARG
    odd = dmel.HmlpWeights(16, 16, 16, 32, *([vp((1 << 20) + 4)] + [a] * 13))
    assert H(a, 1, 40, 40, ctypes.byref(odd), a, a, 1 << 30, None) == dmel.DMEL_ERR_INVALID_ARG
    # no workspace for a real request
    assert H(a, 1, 40, 40, ctypes.byref(w), a, None, 0, None) == dmel.DMEL_ERR_INVALID_ARG
    # the workspace grows with the patch count and covers the fp32 stage outputs
    n1 = lib.dmel_hmlp_workspace_size(1, ctypes.byref(w))
    n10 = lib.dmel_hmlp_workspace_size(10, ctypes.byref(w))
    assert 0 < n1 < n10 and n10 >= 10 * 64 * 16 * 4
    assert lib.dmel_hmlp_workspace_size(0, ctypes.byref(w)) == 0
    # d1 a multiple of 256 (at most 1536): stage 1 runs fused and needs neither the gathered
    # blocks nor the fp32 stage-1 sums; a d1 just off that grid takes the general path
    P = 10
    fused = dmel.HmlpWeights(256, 64, 64, 64, *([a] * 14))
    general = dmel.HmlpWeights(264, 64, 64, 64, *([a] * 14))
    too_wide = dmel.HmlpWeights(1792, 64, 64, 64, *([a] * 14))
    nf = lib.dmel_hmlp_workspace_size(P, ctypes.byref(fused))
    ng = lib.dmel_hmlp_workspace_size(P, ctypes.byref(general))
    nw = lib.dmel_hmlp_workspace_size(P, ctypes.byref(too_wide))
    assert ng - nf >= P * 64 * 256 * 2  # more than half the fp32 stage-1 sums the general path keeps
    assert nw >= nf + P * 64 * 1792 * 4  # past 1536 columns the fp32 sums are back
    # no image: a no-op
    assert H(None, 0, 40, 40, ctypes.byref(w), None, None, 0, None) == dmel.DMEL_OK


def test_table_prepare_size_and_argument_checks_without_gpu(lib):
    """A prepared table (its Gram matrix G, 1280 x 1280 fp32 and a second partial product) exists
    for bf16 tables whose width the tensor-core path tiles, and for nothing else; bad pointers and
    sizes are rejected before any device call."""
    vp = ctypes.c_void_p
    a = vp(1 << 20)
    n = dmel.dmel_table_prepare_size(6144, dmel.DMEL_BF16)
    assert n >= 2 * 1280 * 1280 * 4
    assert dmel.dmel_table_prepare_size(256, dmel.DMEL_BF16) == n
    assert dmel.dmel_table_prepare_size(6144, dmel.DMEL_F32) == 0
    assert dmel.dmel_table_prepare_size(200, dmel.DMEL_BF16) == 0
    assert dmel.dmel_table_prepare_size(0, dmel.DMEL_BF16) == 0
    P = lib.dmel_table_prepare
    assert P(a, 6144, dmel.DMEL_BF16, a, n - 1, None) == dmel.DMEL_ERR_INVALID_ARG  # too small
    assert P(a, 6144, dmel.DMEL_BF16, vp((1 << 20) + 16), n, None) == dmel.DMEL_ERR_INVALID_ARG  # misaligned
    assert P(a, 6144, dmel.DMEL_BF16, None, n, None) == dmel.DMEL_ERR_INVALID_ARG
    assert P(None, 6144, dmel.DMEL_BF16, a, n, None) == dmel.DMEL_ERR_INVALID_ARG
    assert P(a, 6144, dmel.DMEL_F32, a, n, None) == dmel.DMEL_ERR_INVALID_ARG  # no G for fp32 tables
    # a prepared pointer off its 256-byte alignment is an argument error in both calls
    odd = vp((1 << 20) + 64)
    ws_n = dmel.dmel_workspace_size(1000, 6144, dmel.DMEL_BF16, True, True)
    E = lib.dmel_embed_prepared
    assert E(a, 1000, a, dmel.DMEL_BF16, 6144, a, 1e-6, odd, a, dmel.DMEL_BF16, a, ws_n,
             None) == dmel.DMEL_ERR_INVALID_ARG
    ws_f = dmel.dmel_workspace_size(1000, 6144, dmel.DMEL_BF16, True, False)
    Fw = lib.dmel_forward_prepared
    assert Fw(a, a, a, 1, 1000, None, None, a, dmel.DMEL_BF16, 6144, a, 1e-6, odd, a, dmel.DMEL_BF16, None, a, ws_f,
              None) == dmel.DMEL_ERR_INVALID_ARG
    # and a prepared pointer does not relax the other checks
    assert E(a, 1000, a, dmel.DMEL_BF16, 6144, a, 1e-6, a, a, dmel.DMEL_BF16, None, 0,
             None) == dmel.DMEL_ERR_INVALID_ARG
