"""Pins for the CPU oracle: each test checks it against something other than itself.

Sources of truth used here: the constants printed in "Inside Inkling: Audio Design"
(Part 1 · Modeling), library routines that compute the same textbook objects (scipy's periodic
Hann window, numpy's FFT, the HTK filterbanks of transformers and torchaudio, torch's RMSNorm),
closed forms (a bin-centred tone under a Hann window, Parseval, the one-level gain shift) and
brute force on tiny tables.
"""
import json
import os

import numpy as np
import pytest

from encoder_free_audio_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")


def _frame_of(x, t):
    """Raw samples of frame t of a clip under the causal framing (zeros before the clip)."""
    idx = np.arange(800 * (t - 1), 800 * (t + 1))
    out = np.zeros(1600, np.float64)
    ok = idx >= 0
    out[ok] = x[idx[ok]]
    return out


# ---------------------------------------------------------------- page constants (golden)

def test_page_constants(oracle_mod):
    g = json.load(open(GOLDEN))
    o = oracle_mod
    assert g["sample_rate_hz"] // g["hop_samples"] == g["tokens_per_second"]
    assert o.HOP == g["hop_samples"] and o.WIN == g["window_samples"]
    assert o.NMEL == g["n_mel_bins"] and o.NLEV == g["mel_vocab_size"]
    assert o.NMEL * o.NLEV == g["table_rows"]
    assert round(g["table_rows"] * g["table_dim"] / 1e6, 1) == g["table_weights_rounded_millions"]
    # 20 frames per second of audio, 24k frames for a 20-minute clip
    for sec in (1, 2, 10, 30, 60):
        assert o.frames_for_length(g["sample_rate_hz"] * sec) == g["tokens_per_second"] * sec
    assert o.frames_for_length(g["max_clip_minutes"] * 60 * g["sample_rate_hz"]) == g["tokens_for_max_clip"]
    # the clamp ends
    assert o.log_clamp(0.0) == g["dmel_min_value"]
    assert o.log_clamp(1e30) == g["dmel_max_value"]


def test_frame_count_edges(oracle_mod):
    o = oracle_mod
    assert [o.frames_for_length(n) for n in (0, 1, 799, 800, 801, 1599, 1600)] == [0, 0, 0, 1, 1, 1, 2]
    assert o.frames_for_length(-1) == -1
    fo = o.frame_offsets(np.array([0, 799, 2399, 2399, 4000]))
    assert fo.tolist() == [0, 0, 2, 2, 4]
    with pytest.raises(ValueError):
        o.frame_offsets(np.array([0, 900, 800]))
    with pytest.raises(ValueError):
        o.frame_offsets(np.array([5, 900]))


# ---------------------------------------------------------------- window and DFT

def test_window_is_scipy_periodic_hann(oracle_mod):
    from scipy.signal import get_window
    w = oracle_mod.window()
    ref = get_window("hann", 1600, fftbins=True)
    np.testing.assert_allclose(w, ref, rtol=0, atol=1e-15)
    assert abs(w.sum() - 800.0) < 1e-9
    assert abs((w * w).sum() - 600.0) < 1e-9


def test_power_matches_numpy_rfft(oracle_mod):
    from scipy.signal import get_window
    r = np.random.default_rng(3)
    w = get_window("hann", 1600, fftbins=True)
    for scale in (1e-4, 0.3, 1.0):
        fr = r.uniform(-scale, scale, 1600)
        ref = np.abs(np.fft.rfft(w * fr)) ** 2
        P = oracle_mod.power(fr)
        assert P.shape == (801,)
        np.testing.assert_allclose(P, ref, rtol=1e-9, atol=1e-11 * ref.max())


@pytest.mark.parametrize("k0,A,phi", [(2, 1.0, 0.0), (100, 0.5, 1.1), (437, 0.25, -2.0), (798, 0.9, 3.0)])
def test_closed_form_tone(oracle_mod, k0, A, phi):
    """A cos(2 pi k0 n / 1600 + phi) under a periodic Hann window: P_k0 = (400 A)^2,
    P_{k0 +- 1} = (200 A)^2, every other bin zero, for any phase."""
    n = np.arange(1600)
    P = oracle_mod.power(A * np.cos(2 * np.pi * k0 * n / 1600 + phi))
    peak = (400 * A) ** 2
    assert abs(P[k0] - peak) < 1e-9 * peak
    assert abs(P[k0 - 1] - (200 * A) ** 2) < 1e-9 * peak
    assert abs(P[k0 + 1] - (200 * A) ** 2) < 1e-9 * peak
    rest = np.delete(P, [k0 - 1, k0, k0 + 1])
    assert rest.max() < 1e-12 * peak


def test_parseval(oracle_mod):
    r = np.random.default_rng(4)
    w = oracle_mod.window()
    for _ in range(3):
        fr = r.standard_normal(1600)
        P = oracle_mod.power(fr)
        lhs = P[0] + 2 * P[1:800].sum() + P[800]
        rhs = 1600 * np.sum((w * fr) ** 2)
        assert abs(lhs - rhs) < 1e-10 * rhs


# ---------------------------------------------------------------- mel filterbank

def test_htk_mel_scale_textbook(oracle_mod):
    # the HTK scale puts 1000 Hz at (very nearly) 1000 mel
    assert abs(oracle_mod.hz_to_mel(1000.0) - 1000.0) < 0.05
    for f in (0.0, 123.4, 1000.0, 8000.0):
        assert abs(oracle_mod.mel_to_hz(oracle_mod.hz_to_mel(f)) - f) < 1e-9


def test_filterbank_matches_transformers_htk(oracle_mod):
    from transformers.audio_utils import mel_filter_bank
    ref = mel_filter_bank(num_frequency_bins=801, num_mel_filters=80, min_frequency=0.0, max_frequency=8000.0,
                          sampling_rate=16000, norm=None, mel_scale="htk")
    fb = oracle_mod.filterbank()
    assert ref.shape == (801, 80)
    np.testing.assert_allclose(fb, ref.T, rtol=0, atol=1e-12)


def test_filterbank_matches_torchaudio_htk(oracle_mod):
    import torchaudio.functional as AF
    ref = AF.melscale_fbanks(n_freqs=801, f_min=0.0, f_max=8000.0, n_mels=80, sample_rate=16000, norm=None,
                             mel_scale="htk").double().numpy()
    np.testing.assert_allclose(oracle_mod.filterbank(), ref.T, rtol=0, atol=2e-5)


def test_filterbank_partition_of_unity(oracle_mod):
    """Adjacent triangles share their points, so between the peak of the first filter and the
    peak of the last one the 80 weights at every bin add up to 1."""
    fb = oracle_mod.filterbank()
    pk_first = np.argmax(fb[0])
    pk_last = np.argmax(fb[79])
    s = fb[:, pk_first + 1:pk_last].sum(axis=0)  # bins strictly between the two peaks
    np.testing.assert_allclose(s, 1.0, atol=1e-12)
    assert (fb >= 0).all() and fb.max() <= 1.0 + 1e-12
    assert (fb.sum(axis=1) > 0).all()  # no empty filter at 10 Hz bin spacing


def test_tone_lights_expected_mel_bin(oracle_mod):
    """A bin-centred tone at the peak bin of filter b (taken from the transformers filterbank)
    gives its largest mel energy in channel b, for every channel wider than the Hann main lobe."""
    from transformers.audio_utils import mel_filter_bank
    ref = mel_filter_bank(num_frequency_bins=801, num_mel_filters=80, min_frequency=0.0, max_frequency=8000.0,
                          sampling_rate=16000, norm=None, mel_scale="htk")
    n = np.arange(1600)
    for b in range(10, 80):
        k = int(np.argmax(ref[:, b]))
        M = oracle_mod.mel(0.5 * np.cos(2 * np.pi * k * n / 1600))
        assert int(np.argmax(M)) == b, (b, k)


# ---------------------------------------------------------------- log, clamp, quantise

def test_quantiser_levels(oracle_mod):
    o = oracle_mod
    for k in range(16):
        lo = -7.0 + 9.0 * k / 16
        hi = -7.0 + 9.0 * (k + 1) / 16
        assert o.quantise(lo + 1e-9) == k
        assert o.quantise(0.5 * (lo + hi)) == k
        if k < 15:
            assert o.quantise(hi - 1e-9) == k
    assert o.quantise(-7.0) == 0
    assert o.quantise(2.0) == 15
    assert o.log_clamp(0.0) == -7.0
    assert o.log_clamp(float("nan")) == -7.0
    assert o.log_clamp(float("inf")) == 2.0
    assert o.log_clamp(-5.0) == -7.0
    assert abs(o.log_clamp(1e-3) - (-3.0)) < 1e-15
    assert o.log_clamp(1e5) == 2.0


def test_silence_codes_zero(oracle_mod):
    wav = np.zeros(16000, np.float32)
    c, lh = oracle_mod.codes(wav, np.array([0, 16000]))
    assert c.shape == (20, 80)
    assert (c == 0).all() and (lh == -7.0).all()


def test_full_scale_noise_reaches_top_level(oracle_mod):
    r = np.random.default_rng(5)
    wav = np.where(r.random(16000 * 4) < 0.5, -1.0, 1.0).astype(np.float32)
    c = oracle_mod.codes(wav, np.array([0, wav.size]), want_lhat=False)
    assert (c[1:] == 15).mean() >= 0.99  # frame 0 is half zeros
    n = np.arange(1600 * 4)
    tone = np.cos(2 * np.pi * 100 * n / 1600).astype(np.float32)  # 1 kHz, bin-centred, full scale
    c2 = oracle_mod.codes(tone, np.array([0, tone.size]), want_lhat=False)
    fb = oracle_mod.filterbank()
    b = int(np.argmax(fb[:, 100]))
    assert (c2[1:, b] == 15).all()


def test_gain_shift_is_one_level(oracle_mod):
    """x -> x * 10^(9/32) multiplies every energy by 10^(9/16), i.e. adds 0.5625 (one level) to L."""
    wav, off = synth.one_clip_2s()
    g = 10.0 ** (9.0 / 32.0)
    c0, l0 = oracle_mod.codes(wav, off)
    c1, l1 = oracle_mod.codes((wav.astype(np.float64) * g).astype(np.float32), off)
    inner = (l0 > -7.0 + 1e-6) & (l0 < 2.0 - 0.5625 - 1e-6)
    assert inner.sum() > 500
    # fp32 rounding of the scaled input perturbs L by ~1e-7
    assert np.max(np.abs((l1 - l0)[inner] - 0.5625)) < 1e-5
    safe = inner & (oracle_mod.boundary_distance(l0) > 1e-4)
    assert (c1[safe].astype(int) - c0[safe].astype(int) == 1).all()


def test_nonfinite_samples_give_valid_codes(oracle_mod):
    wav = np.zeros(8000, np.float32)
    wav[1000] = np.nan
    wav[5000] = np.inf
    c = oracle_mod.codes(wav, np.array([0, 8000]), want_lhat=False)
    assert c.shape == (10, 80) and c.max() <= 15


# ---------------------------------------------------------------- framing: streaming and ragged

def test_streaming_equals_offline(oracle_mod):
    wav, off = synth.one_clip_2s()
    full = oracle_mod.codes(wav, off, want_lhat=False)
    tail = np.zeros((1, 800), np.float32)
    got = []
    for k in range(40):
        piece = wav[800 * k:800 * (k + 1)]
        got.append(oracle_mod.codes(piece, np.array([0, 800]), tails=tail, want_lhat=False))
        tail = oracle_mod.tails_out(piece, np.array([0, 800]), tails=tail)
    np.testing.assert_array_equal(np.concatenate(got), full)


def test_tail_out_rules(oracle_mod):
    x = np.arange(2000, dtype=np.float32)
    t_in = -np.ones((1, 800), np.float32)
    out = oracle_mod.tails_out(x, np.array([0, 2000]), tails=t_in)
    np.testing.assert_array_equal(out[0], x[800:1600])  # F = 2: samples [800, 1600)
    out0 = oracle_mod.tails_out(x[:500], np.array([0, 500]), tails=t_in)
    np.testing.assert_array_equal(out0[0], t_in[0])  # F = 0: tail passes through


def test_ragged_equals_per_clip(oracle_mod):
    r = np.random.default_rng(6)
    lengths = [800, 0, 2399, 799, 5000, 1600]
    off = synth.offsets_from_lengths(lengths)
    wav = r.uniform(-0.5, 0.5, int(off[-1])).astype(np.float32)
    allc = oracle_mod.codes(wav, off, want_lhat=False)
    fo = oracle_mod.frame_offsets(off)
    for c, n in enumerate(lengths):
        one = oracle_mod.codes(wav[off[c]:off[c + 1]], np.array([0, n]), want_lhat=False)
        np.testing.assert_array_equal(allc[fo[c]:fo[c + 1]], one)


def test_frame_subset_equals_full_run(oracle_mod):
    wav, off = synth.one_clip_2s()
    full = oracle_mod.codes(wav, off, want_lhat=False)
    ids = np.array([39, 0, 17, 17, 5])
    np.testing.assert_array_equal(oracle_mod.codes(wav, off, frame_ids=ids, want_lhat=False), full[ids])
    with pytest.raises(ValueError):
        oracle_mod.codes(wav, off, frame_ids=np.array([40]))


def test_thread_count_changes_nothing(oracle_mod):
    """The oracle's threads split frames only: one thread and all threads give bit-identical
    codes, log-mel values and embeddings (the host baseline times both)."""
    wav, off = synth.one_clip_2s()
    table = np.random.default_rng(9).standard_normal((1280, 16))
    n_all = oracle_mod.threads()
    c_all, l_all = oracle_mod.codes(wav, off)
    e_all = oracle_mod.embed(c_all, table, np.ones(16))
    try:
        assert oracle_mod.set_threads(1) == 1
        c_one, l_one = oracle_mod.codes(wav, off)
        e_one = oracle_mod.embed(c_one, table, np.ones(16))
    finally:
        assert oracle_mod.set_threads(n_all) == n_all
    np.testing.assert_array_equal(c_one, c_all)
    np.testing.assert_array_equal(l_one, l_all)
    np.testing.assert_array_equal(e_one, e_all)


def test_frame_alignment_closed_form(oracle_mod):
    """Frame t of a clip sees samples [800 (t - 1), 800 (t + 1)): a clip that is silent except
    for a bin-centred tone in [800 t0, 800 t0 + 800) lights frames t0 and t0 + 1 only."""
    x = np.zeros(8000, np.float32)
    t0 = 4
    n = np.arange(800)
    x[800 * t0:800 * t0 + 800] = np.cos(2 * np.pi * 100 * n / 1600)
    c = oracle_mod.codes(x, np.array([0, 8000]), want_lhat=False)
    lit = np.where(c.max(axis=1) > 0)[0].tolist()
    assert lit == [t0, t0 + 1]
    # and the oracle's frame equals a direct slice under the same rule
    P = oracle_mod.power(_frame_of(x.astype(np.float64), t0))
    assert P.max() > 1e3


# ---------------------------------------------------------------- embedding and RMSNorm

def test_embed_bruteforce_tiny_integer_table(oracle_mod):
    r = np.random.default_rng(7)
    dim = 8
    T = r.integers(-8, 9, size=(1280, dim)).astype(np.float64)
    codes = r.integers(0, 16, size=(5, 80)).astype(np.uint8)
    got = oracle_mod.embed(codes, T)
    for f in range(5):
        for j in range(dim):
            s = 0
            for b in range(80):
                s += int(T[16 * b + int(codes[f, b]), j])
            assert got[f, j] == s
    # a row layout 16 * c + b (transposed) would give a different answer
    alt = np.array([[sum(T[16 * int(codes[f, b]) % 1280 + b, j] for b in range(80)) for j in range(dim)]
                    for f in range(5)])
    assert not np.array_equal(alt, got)


def test_embed_order_invariance(oracle_mod):
    """The sum does not depend on which bin is added first: permuting bins together with the
    table's 16-row blocks leaves every frame vector unchanged."""
    r = np.random.default_rng(8)
    T = r.normal(0, 0.02, (1280, 16))
    codes = r.integers(0, 16, size=(7, 80)).astype(np.uint8)
    perm = r.permutation(80)
    Tp = T.reshape(80, 16, 16)[perm].reshape(1280, 16)
    a = oracle_mod.embed(codes, T)
    b = oracle_mod.embed(codes[:, perm], Tp)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-15)


def test_rmsnorm_closed_form(oracle_mod):
    c = 0.0125
    T = np.full((1280, 24), c)
    g = np.linspace(0.5, 1.5, 24)
    codes = np.random.default_rng(9).integers(0, 16, size=(3, 80)).astype(np.uint8)
    y = oracle_mod.embed(codes, T, g, eps=1e-6)
    x = 80 * c
    np.testing.assert_allclose(y, np.broadcast_to(g * x / np.sqrt(x * x + 1e-6), y.shape), rtol=1e-14)


def test_rmsnorm_matches_torch(oracle_mod):
    import torch
    r = np.random.default_rng(10)
    T = r.normal(0, 0.02, (1280, 64))
    g = r.normal(1, 0.1, 64)
    codes = r.integers(0, 16, size=(6, 80)).astype(np.uint8)
    x = oracle_mod.embed(codes, T)
    y = oracle_mod.embed(codes, T, g, eps=1e-6)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(g), eps=1e-6).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=0)


def test_embed_rejects_bad_code(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.embed(np.full((1, 80), 16, np.uint8), np.zeros((1280, 8)))


# ---------------------------------------------------------------- sentinel expansion (splice)

SPLICE_GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "splice_example.json")


def test_splice_hand_worked_example(oracle_mod):
    g = json.load(open(SPLICE_GOLDEN))
    token_pos, frame_rows, n, audio = oracle_mod.splice_plan(g["seq_len"], g["sentinel_pos"], g["frames_per_item"])
    assert token_pos == g["token_pos"] and frame_rows == g["frame_rows"]
    assert n == g["expanded_len"] and audio == g["audio_tokens"]


@pytest.mark.parametrize("seed", range(6))
def test_splice_closed_forms(oracle_mod, seed):
    r = np.random.default_rng(500 + seed)
    seq_len = int(r.integers(1, 60))
    k = int(r.integers(0, seq_len + 1))
    pos = sorted(r.choice(seq_len, size=k, replace=False).tolist())
    f = r.integers(0, 9, size=k).tolist()
    token_pos, frame_rows, n, audio = oracle_mod.splice_plan(seq_len, pos, f)
    # each sentinel gives way to its f frames: the sequence grows by sum(f - 1)
    assert n == seq_len + sum(x - 1 for x in f) and audio == sum(f)
    # every expanded position is used exactly once, by a surviving token or a frame
    used = [p for p in token_pos if p >= 0] + frame_rows
    assert sorted(used) == list(range(n))
    # tokens keep their order, a token before a sentinel keeps its index, and a token moves by
    # the frames minus sentinels in front of it
    survivors = [(p, q) for p, q in enumerate(token_pos) if q >= 0]
    assert all(a[1] < b[1] for a, b in zip(survivors, survivors[1:]))
    for p, q in survivors:
        before = [i for i, s in enumerate(pos) if s < p]
        assert q == p + sum(f[i] - 1 for i in before)
    # an item's frames are consecutive and start where its sentinel stood (shifted)
    starts = np.concatenate([[0], np.cumsum(f)]).astype(int)
    for i, s in enumerate(pos):
        rows = frame_rows[starts[i]:starts[i + 1]]
        assert rows == list(range(rows[0], rows[0] + f[i])) if f[i] else rows == []
        if f[i]:
            assert rows[0] == s + sum(f[j] - 1 for j in range(i))


def test_splice_special_cases(oracle_mod):
    # no sentinel: the identity
    tp, fr, n, a = oracle_mod.splice_plan(5, [], [])
    assert tp == [0, 1, 2, 3, 4] and fr == [] and n == 5 and a == 0
    # clips with no frame: their sentinels vanish
    tp, fr, n, a = oracle_mod.splice_plan(4, [0, 2], [0, 0])
    assert tp == [-1, 0, -1, 1] and fr == [] and n == 2 and a == 0
    # an audio-only request: one sentinel, 20 frames per second of audio
    tp, fr, n, a = oracle_mod.splice_plan(1, [0], [40])
    assert tp == [-1] and fr == list(range(40)) and n == 40 and a == 40


# ---------------------------------------------------------------- quantiser variants

SERVE_CLAMP = (-1.5, 2.0)  # the serving default's minimum ("Inside Inkling: Audio Design", Coda)


def test_quant_default_variant_is_the_default(oracle_mod):
    wav, off = synth.one_clip_2s()
    c0, l0 = oracle_mod.codes(wav, off)
    c1, l1 = oracle_mod.codes_q(wav, off, oracle_mod.DEFAULT_QUANT)
    assert (c0 == c1).all() and (l0 == l1).all()


def test_quant_round_is_nearest_reconstruction_point(oracle_mod):
    """Mode 1: brute force over the 16 reconstruction points lmin + k (lmax - lmin) / 15."""
    for lmin, lmax in ((-7.0, 2.0), SERVE_CLAMP):
        pts = lmin + (lmax - lmin) * np.arange(16) / 15.0
        for k, p in enumerate(pts):
            assert oracle_mod.quantise_q(p, lmin, lmax, 1) == k
        r = np.random.default_rng(11)
        for L in r.uniform(lmin, lmax, 3000):
            d = np.abs(L - pts)
            if np.sort(d)[1] - d.min() < 1e-9:
                continue  # a tie between two points
            assert oracle_mod.quantise_q(L, lmin, lmax, 1) == int(np.argmin(d))


def test_quant_mulaw_matches_library_companding(oracle_mod):
    """Mode 2: numpy's log1p companding of u = (L - lmin) / (lmax - lmin), then 16 levels."""
    mu = 255.0
    for lmin, lmax in ((-7.0, 2.0), SERVE_CLAMP):
        r = np.random.default_rng(12)
        Ls = np.concatenate([r.uniform(lmin, lmax, 3000), [lmin, lmax]])
        u = (Ls - lmin) / (lmax - lmin)
        y = 16.0 * np.log1p(mu * u) / np.log1p(mu)
        ref = np.minimum(15, np.floor(y)).astype(int)
        near = np.abs(y - np.round(y)) < 1e-9
        got = np.array([oracle_mod.quantise_q(L, lmin, lmax, 2, mu) for L in Ls])
        assert (got[~near] == ref[~near]).all()
        assert got[-2] == 0 and got[-1] == 15
        # companding spends more levels near the bottom of the range
        assert (got == 0).mean() < 1.0 / 16 and (got == 15).mean() > 1.0 / 16


def test_quant_serving_clamp_special_cases(oracle_mod):
    q = (SERVE_CLAMP[0], SERVE_CLAMP[1], 0, 0.0)
    c, lh = oracle_mod.codes_q(np.zeros(16000, np.float32), np.array([0, 16000]), q)
    assert (c == 0).all() and (lh == -1.5).all()  # silence sits at the new bottom
    r = np.random.default_rng(5)
    wav = np.where(r.random(16000 * 4) < 0.5, -1.0, 1.0).astype(np.float32)
    c, _ = oracle_mod.codes_q(wav, np.array([0, wav.size]), q)
    assert (c[1:] == 15).mean() >= 0.99


def test_quant_serving_clamp_gain_shift_is_one_level(oracle_mod):
    """With the clamp [-1.5, 2] a level is 3.5 / 16 wide: x -> x * 10^(3.5/32) adds one level."""
    q = (SERVE_CLAMP[0], SERVE_CLAMP[1], 0, 0.0)
    w = (SERVE_CLAMP[1] - SERVE_CLAMP[0]) / 16
    wav, off = synth.one_clip_2s()
    g = 10.0 ** (w / 2.0)
    c0, l0 = oracle_mod.codes_q(wav, off, q)
    c1, l1 = oracle_mod.codes_q((wav.astype(np.float64) * g).astype(np.float32), off, q)
    inner = (l0 > SERVE_CLAMP[0] + 1e-6) & (l0 < SERVE_CLAMP[1] - w - 1e-6)
    assert inner.sum() > 300
    assert np.max(np.abs((l1 - l0)[inner] - w)) < 1e-5
    safe = inner & (oracle_mod.boundary_distance_q(l0, q) > 1e-4)
    assert (c1[safe].astype(int) - c0[safe].astype(int) == 1).all()


# ---------------------------------------------------------------- ShortConv (Part 3 · Inference)

def _conv_numpy(x, w, hist):
    """Per channel: numpy's full convolution of [history, x] with (1 + w0, w1, w2, w3), cut to
    the positions of x (a library routine for the same causal filter)."""
    T, C = x.shape
    out = np.zeros((T, C))
    for c in range(C):
        h = np.array([1.0 + w[c, 0], w[c, 1], w[c, 2], w[c, 3]])
        full = np.convolve(np.concatenate([hist[:, c], x[:, c]]), h)
        out[:, c] = full[3:3 + T]
    return out


def test_shortconv_matches_numpy_convolution(oracle_mod):
    r = np.random.default_rng(21)
    C = 24
    lens = [0, 1, 2, 3, 17, 5]
    off = np.concatenate([[0], np.cumsum(lens)])
    x = r.standard_normal((off[-1], C))
    w = r.standard_normal((C, 4))
    st = r.standard_normal((len(lens), 3, C))
    y, so = oracle_mod.shortconv(x, off, w, st)
    for s, T in enumerate(lens):
        seg = x[off[s]:off[s + 1]]
        np.testing.assert_allclose(y[off[s]:off[s + 1]], _conv_numpy(seg, w, st[s]), rtol=1e-12, atol=1e-12)
        full = np.concatenate([st[s], seg])
        np.testing.assert_array_equal(so[s], full[-3:])


def test_shortconv_impulse_response_and_identity(oracle_mod):
    C = 8
    w = np.arange(C * 4, dtype=np.float64).reshape(C, 4) / 10.0
    x = np.zeros((10, C))
    x[4] = 1.0
    y, _ = oracle_mod.shortconv(x, [0, 10], w)
    # the impulse reappears with gain 1 + w0 at its own step and w_d d steps later
    expect = np.zeros((10, C))
    expect[4] = 1.0 + w[:, 0]
    for d in (1, 2, 3):
        expect[4 + d] = w[:, d]
    np.testing.assert_array_equal(y, expect)
    y0, _ = oracle_mod.shortconv(np.random.default_rng(2).standard_normal((7, C)), [0, 7], np.zeros((C, 4)))
    x0 = np.random.default_rng(2).standard_normal((7, C))
    np.testing.assert_array_equal(y0, x0)  # zero weights: the identity


def test_shortconv_streaming_equals_offline(oracle_mod):
    """Decoding token by token (or in chunks) with the carried state gives the offline result."""
    r = np.random.default_rng(23)
    C, T = 16, 29
    x = r.standard_normal((T, C))
    w = r.standard_normal((C, 4))
    y_all, s_all = oracle_mod.shortconv(x, [0, T], w)
    st = np.zeros((1, 3, C))
    ys = []
    for a, b in ((0, 1), (1, 2), (2, 9), (9, 9), (9, 10), (10, 29)):
        yc, st = oracle_mod.shortconv(x[a:b], [0, b - a], w, st)
        ys.append(yc)
    np.testing.assert_allclose(np.concatenate(ys), y_all, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(st, s_all)


# ---------------------------------------------------------------- hMLP patchifier

def _hmlp_params(r, d1, d2, d3, D):
    p = {"W1": r.standard_normal((75, d1)) / np.sqrt(75), "b1": 0.1 * r.standard_normal(d1),
         "g1": 1 + 0.1 * r.standard_normal(d1), "be1": 0.1 * r.standard_normal(d1),
         "W2": r.standard_normal((4 * d1, d2)) / np.sqrt(4 * d1), "b2": 0.1 * r.standard_normal(d2),
         "g2": 1 + 0.1 * r.standard_normal(d2), "be2": 0.1 * r.standard_normal(d2),
         "W3": r.standard_normal((4 * d2, d3)) / np.sqrt(4 * d2), "b3": 0.1 * r.standard_normal(d3),
         "g3": 1 + 0.1 * r.standard_normal(d3), "be3": 0.1 * r.standard_normal(d3),
         "W4": r.standard_normal((4 * d3, D)) / np.sqrt(4 * d3), "b4": 0.1 * r.standard_normal(D)}
    return p


def test_hmlp_matches_strided_convolutions(oracle_mod):
    """The hMLP as torch's conv2d with kernel = stride (5, 2, 2, 2), layer norm over channels and
    the exact GELU, bf16 storage between stages: an independent formulation on the image grid."""
    import torch
    import torch.nn.functional as Fn
    r = np.random.default_rng(31)
    d1, d2, d3, D = 8, 12, 16, 24
    p = _hmlp_params(r, d1, d2, d3, D)
    img = oracle_mod._bf16(r.uniform(-1, 1, (2, 80, 120, 3)))
    got = oracle_mod.hmlp(img, p)
    x = torch.from_numpy(img).permute(0, 3, 1, 2)  # NCHW, float64
    # stage 1 weight: row (5 kr + kc) * 3 + ch of W1 -> conv weight [out, ch, kr, kc]
    w1 = torch.from_numpy(p["W1"].reshape(5, 5, 3, d1)).permute(3, 2, 0, 1)
    def bf(t):
        return torch.from_numpy(oracle_mod._bf16(t.numpy()))
    def ln_gelu(t, g, b):
        t = t.permute(0, 2, 3, 1)
        t = Fn.layer_norm(t, (t.shape[-1],), torch.from_numpy(g), torch.from_numpy(b), eps=1e-6)
        return Fn.gelu(t).permute(0, 3, 1, 2)
    h = bf(ln_gelu(Fn.conv2d(x, w1, torch.from_numpy(p["b1"]), stride=5), p["g1"], p["be1"]))
    for s, d_in in ((2, d1), (3, d2), (4, d3)):
        d_out = p[f"W{s}"].shape[1]
        # rows of Ws: child k = 2 kr + kc (tl, tr, bl, br), then its d_in channels
        ws = torch.from_numpy(p[f"W{s}"].reshape(2, 2, d_in, d_out)).permute(3, 2, 0, 1)
        h = Fn.conv2d(h, ws, torch.from_numpy(p[f"b{s}"]), stride=2)
        h = bf(ln_gelu(h, p[f"g{s}"], p[f"be{s}"]) if s < 4 else h)
    ref = h.permute(0, 2, 3, 1).reshape(-1, D).numpy()  # patches in raster order
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-2 * np.abs(ref).max())
    # away from bf16 rounding ties the two agree to the last bit of the storage type
    assert (np.abs(got - ref) <= 2 ** -7 * np.maximum(np.abs(ref), 1e-3)).mean() > 0.99


def test_hmlp_closed_forms(oracle_mod):
    r = np.random.default_rng(32)
    d1, d2, d3, D = 4, 4, 4, 6
    p = _hmlp_params(r, d1, d2, d3, D)
    p["W4"][:] = 0.0  # the last stage ignores its input: every patch is b4 (rounded to bf16)
    img = r.uniform(-1, 1, (1, 40, 80, 3))
    out = oracle_mod.hmlp(img, p)
    np.testing.assert_array_equal(out, np.tile(oracle_mod._bf16(p["b4"]), (2, 1)))
    # patches are independent: swapping the two 40 x 40 halves swaps the outputs
    p2 = _hmlp_params(r, d1, d2, d3, D)
    a = oracle_mod.hmlp(img, p2)
    b = oracle_mod.hmlp(np.concatenate([img[:, :, 40:], img[:, :, :40]], axis=2), p2)
    np.testing.assert_array_equal(a, b[::-1])
