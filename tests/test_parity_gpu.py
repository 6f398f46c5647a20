"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded
inputs. Codes must match except within 1e-4 of a level boundary (flips are counted and
printed); embeddings within 1e-5 (fp32 output) or 1e-2 (bf16 output) of max(|o_j|, rms(o))."""
import numpy as np
import pytest
import torch

from encoder_free_audio_b200 import build, dmel, synth
from encoder_free_audio_b200.frontend import FrontEnd
from helpers import bf16_table, compare_codes, compare_embed

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    dmel.library()
    dmel.dmel_get_device_error(clear=True)
    yield
    assert dmel.dmel_get_device_error(clear=True) == 0


@pytest.fixture(scope="module")
def table_bf16():
    t, t64 = bf16_table(synth.table())
    return t.to(DEV), t64


@pytest.fixture(scope="module")
def rmsw_bf16():
    g = torch.from_numpy(synth.rms_weight()).to(torch.bfloat16)
    return g.to(DEV), g.float().numpy().astype(np.float64)


def _codes_gpu(wav, off, tails=None, want_tails=False):
    fo = dmel.dmel_frame_offsets(off)
    F = int(fo[-1])
    w = torch.from_numpy(wav).to(DEV)
    so_d = torch.from_numpy(off).to(DEV)
    fo_d = torch.from_numpy(fo).to(DEV)
    codes = torch.empty((F, 80), dtype=torch.uint8, device=DEV)
    t_in = None if tails is None else torch.from_numpy(tails).to(DEV)
    t_out = torch.full((off.shape[0] - 1, 800), -5.0, device=DEV) if want_tails else None
    dmel.dmel_codes(w, so_d, fo_d, F, codes, tails=t_in, tails_out=t_out)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), (None if t_out is None else t_out.cpu().numpy())


# ------------------------------------------------------------------------- codes

def test_codes_one_clip_2s(oracle_mod):
    wav, off = synth.one_clip_2s()
    g, tails = _codes_gpu(wav, off, want_tails=True)
    oc, ol = oracle_mod.codes(wav, off)
    flips, _ = compare_codes(g, oc, ol)
    print(f"one_clip_2s: 40 frames, flips {flips}")
    np.testing.assert_array_equal(tails, oracle_mod.tails_out(wav, off))


def test_codes_edge_lengths_and_tails(oracle_mod):
    r = np.random.default_rng(21)
    lengths = [0, 1, 799, 800, 801, 1599, 1600, 2400, 5 * 800 + 13, 0, 3200]
    off = synth.offsets_from_lengths(lengths)
    wav = r.uniform(-0.7, 0.7, int(off[-1])).astype(np.float32)
    tails = r.uniform(-0.5, 0.5, (len(lengths), 800)).astype(np.float32)
    g, t_out = _codes_gpu(wav, off, tails=tails, want_tails=True)
    oc, ol = oracle_mod.codes(wav, off, tails=tails)
    compare_codes(g, oc, ol)
    np.testing.assert_array_equal(t_out, oracle_mod.tails_out(wav, off, tails))


def test_codes_tails_in_place_and_no_frames(oracle_mod):
    """The carried tails written in place (tails_out = tails: a kernel of their own after the
    codes) equal those written into another buffer (by the codes kernel itself, after each warp's
    frames); a batch with no frame at all passes the tails in through."""
    r = np.random.default_rng(23)
    lengths = [0, 1, 799, 800, 801, 1599, 1600, 2400, 5 * 800 + 13, 0, 3200] * 300
    off = synth.offsets_from_lengths(lengths)
    wav = r.uniform(-0.7, 0.7, int(off[-1])).astype(np.float32)
    tails = r.uniform(-0.5, 0.5, (len(lengths), 800)).astype(np.float32)
    g, t_out = _codes_gpu(wav, off, tails=tails, want_tails=True)
    fo = dmel.dmel_frame_offsets(off)
    F = int(fo[-1])
    codes = torch.empty((F, 80), dtype=torch.uint8, device=DEV)
    t_io = torch.from_numpy(tails).to(DEV)
    dmel.dmel_codes(torch.from_numpy(wav).to(DEV), torch.from_numpy(off).to(DEV), torch.from_numpy(fo).to(DEV), F,
                    codes, tails=t_io, tails_out=t_io)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes.cpu().numpy(), g)
    np.testing.assert_array_equal(t_io.cpu().numpy(), t_out)
    np.testing.assert_array_equal(t_out, oracle_mod.tails_out(wav, off, tails))
    # no frame in the batch: the codes kernel does not run
    off0 = synth.offsets_from_lengths([0, 799, 5, 0])
    w0 = r.uniform(-0.7, 0.7, int(off0[-1])).astype(np.float32)
    tl0 = r.uniform(-0.5, 0.5, (4, 800)).astype(np.float32)
    g0, t0 = _codes_gpu(w0, off0, tails=tl0, want_tails=True)
    assert g0.shape == (0, 80)
    np.testing.assert_array_equal(t0, oracle_mod.tails_out(w0, off0, tl0))


def test_codes_silence_and_full_scale(oracle_mod):
    r = np.random.default_rng(22)
    off = synth.offsets_from_lengths([16000, 16000])
    wav = np.concatenate([np.zeros(16000), np.where(r.random(16000) < 0.5, -1.0, 1.0)]).astype(np.float32)
    g, _ = _codes_gpu(wav, off)
    assert (g[:20] == 0).all()
    oc, ol = oracle_mod.codes(wav, off)
    compare_codes(g, oc, ol)


def test_codes_nonfinite_samples_stay_in_range():
    wav = np.zeros(8000, np.float32)
    wav[1234] = np.nan
    wav[4321] = np.inf
    g, _ = _codes_gpu(wav, np.array([0, 8000]))
    assert g.shape == (10, 80) and g.max() <= 15


def test_codes_no_frames_is_noop():
    wav = np.zeros(500, np.float32)
    off = np.array([0, 500], np.int64)
    g, _ = _codes_gpu(wav, off)
    assert g.shape == (0, 80)


# ---------------------------------------------------------------- codes: quantiser variants

QUANTS = [(-1.5, 2.0, dmel.DMEL_QUANT_FLOOR, 0.0), (-7.0, 2.0, dmel.DMEL_QUANT_ROUND, 0.0),
          (-1.5, 2.0, dmel.DMEL_QUANT_ROUND, 0.0), (-7.0, 2.0, dmel.DMEL_QUANT_MULAW, 255.0),
          (-1.5, 2.0, dmel.DMEL_QUANT_MULAW, 255.0)]


def _codes_q_gpu(wav, off, q):
    fo = dmel.dmel_frame_offsets(off)
    F = int(fo[-1])
    codes = torch.empty((F, 80), dtype=torch.uint8, device=DEV)
    dmel.dmel_codes_q(torch.from_numpy(wav).to(DEV), torch.from_numpy(off).to(DEV), torch.from_numpy(fo).to(DEV), F,
                      codes, quantizer=q)
    torch.cuda.synchronize()
    return codes.cpu().numpy()


def test_codes_q_default_is_dmel_codes():
    wav, off = synth.batch64_10s(n_clips=16)
    base, _ = _codes_gpu(wav, off)
    assert (_codes_q_gpu(wav, off, None) == base).all()
    assert (_codes_q_gpu(wav, off, (-7.0, 2.0, dmel.DMEL_QUANT_FLOOR, 0.0)) == base).all()


@pytest.mark.parametrize("q", QUANTS)
def test_codes_q_variants_match_oracle(q, oracle_mod):
    """The level mappings the pages leave open, on 16 clips of the batch workload (3,200 frames:
    silence, clipped full scale, pink noise and chirps): equal to the oracle's codes except where
    the oracle's log-mel value lies within 1e-4 of one of the variant's own boundaries."""
    wav, off = synth.batch64_10s(n_clips=16)
    got = _codes_q_gpu(wav, off, q)
    oc, ol = oracle_mod.codes_q(wav, off, q)
    flips, _ = compare_codes(got, oc, ol, boundaries=oracle_mod.level_boundaries_q(*q))
    print(f"quantiser {q}: {flips} boundary flips of {oc.size} cells")


# ------------------------------------------------------------------------- embedding

@pytest.mark.parametrize("dim", [8, 24, 1000, 256, 512])
@pytest.mark.parametrize("tdt", ["f32", "bf16"])
def test_embed_small_integer_tables_exact(dim, tdt, oracle_mod):
    """Tables of small integers: every partial sum is exact in fp32, so the CUDA-core path and
    the tensor-core path (bf16, D % 256 == 0) must give the oracle's sums bit for bit."""
    r = np.random.default_rng(30 + dim)
    T = r.integers(-6, 7, size=(1280, dim)).astype(np.float32)
    F = 300  # 2 full tiles of 128 frames and a ragged tail of 44
    codes = synth.random_codes(31, F)
    tt = torch.from_numpy(T).to(DEV)
    if tdt == "bf16":
        tt = tt.to(torch.bfloat16)
    out = torch.empty((F, dim), dtype=torch.float32, device=DEV)
    dmel.dmel_embed(torch.from_numpy(codes).to(DEV), tt, out)
    torch.cuda.synchronize()
    ref = oracle_mod.embed(codes, T.astype(np.float64))
    np.testing.assert_array_equal(out.cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("out_dt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rms", [False, True])
def test_embed_tensor_core_model_dim(out_dt, rms, table_bf16, rmsw_bf16, oracle_mod):
    T, T64 = table_bf16
    g, g64 = rmsw_bf16
    F = 1000
    codes = synth.random_codes(41, F)
    out = torch.empty((F, 6144), dtype=out_dt, device=DEV)
    ws_n = dmel.dmel_workspace_size(F, 6144, dmel.DMEL_BF16, rms, True)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=DEV)
    dmel.dmel_embed(torch.from_numpy(codes).to(DEV), T, out, rms_weight=g if rms else None, eps=1e-6, workspace=ws)
    torch.cuda.synchronize()
    ref = oracle_mod.embed(codes, T64, g64 if rms else None, 1e-6)
    worst = compare_embed(out.float().cpu().numpy(), ref, 1e-5 if out_dt == torch.float32 else 1e-2)
    print(f"tensor-core embed out={out_dt} rms={rms}: worst {worst:.2e}")


@pytest.mark.parametrize("dim", [256, 768, 2048, 4096, 7168])
def test_embed_tensor_core_rmsnorm_widths(dim, oracle_mod):
    """Fused RMSNorm where a frame tile's row sums come from several column slices, and a ragged
    last frame tile. Resident-table kernel: slices of 32 columns on 8, 24 and 64 clusters (256,
    768, 2048), 64 and 32 (4096), and 7168, whose slices would be wider than the table space
    allows, falls back to the streamed kernel; streamed sparse kernel: 192-column tiles, partial
    last tiles included; dense kernels: 1, 3, 8, 16 and 28 tiles of 256."""
    T, T64 = bf16_table(synth.table(seed=12, dim=dim))
    gw = torch.from_numpy(synth.rms_weight(seed=13, dim=dim)).to(torch.bfloat16)
    F = 700
    codes = synth.random_codes(43, F)
    out = torch.empty((F, dim), dtype=torch.float32, device=DEV)
    ws = torch.empty(dmel.dmel_workspace_size(F, dim, dmel.DMEL_BF16, True, True), dtype=torch.uint8, device=DEV)
    dmel.dmel_embed(torch.from_numpy(codes).to(DEV), T.to(DEV), out, rms_weight=gw.to(DEV), eps=1e-6, workspace=ws)
    torch.cuda.synchronize()
    ref = oracle_mod.embed(codes, T64, gw.float().numpy().astype(np.float64), 1e-6)
    compare_embed(out.cpu().numpy(), ref, 1e-5)


@pytest.mark.parametrize("dim", [128, 6144])
def test_gram_matrix_of_the_table(dim):
    """G = T T^T on the tensor cores (bf16 products, fp32 sums) against the exact product of the
    same bf16 values, on the 55 upper 128 x 128 blocks the RMSNorm scales read."""
    T, T64 = bf16_table(synth.table(seed=21, dim=dim))
    G = torch.full((2, 1280, 1280), float("nan"), dtype=torch.float32, device=DEV)
    dmel.dmel_debug_gram(T.to(DEV), G)
    torch.cuda.synchronize()
    got = G[0].cpu().numpy().astype(np.float64)
    ref = T64 @ T64.T
    # off the diagonal: the tensor cores' fp32 sums of `dim` products; on it: fp64 sums rounded once
    tol = 4e-5 * np.sqrt(np.outer(np.diag(ref), np.diag(ref)))
    assert (np.abs(np.diag(got) - np.diag(ref)) <= 1e-7 * np.diag(ref)).all()
    for g in range(10):
        for h in range(g, 10):
            blk = (slice(128 * g, 128 * g + 128), slice(128 * h, 128 * h + 128))
            assert np.isfinite(got[blk]).all()
            assert (np.abs(got[blk] - ref[blk]) <= tol[blk]).all(), (g, h)


def test_embed_rmsnorm_from_gram_matches_oracle(table_bf16, rmsw_bf16, oracle_mod):
    """The RMSNorm scales from G (the path of calls of 16,384 frames or more) match the oracle at
    fp32 output, ragged last tile; the exchange of row sums inside the kernel, which smaller calls
    take, is checked by the other tests here and under DMEL_EMBED_NORM=exchange."""
    T, T64 = table_bf16
    g, g64 = rmsw_bf16
    F = 16384 + 333
    codes = synth.random_codes(44, F)
    out = torch.empty((F, 6144), dtype=torch.float32, device=DEV)
    ws = torch.empty(dmel.dmel_workspace_size(F, 6144, dmel.DMEL_BF16, True, True), dtype=torch.uint8, device=DEV)
    dmel.dmel_embed(torch.from_numpy(codes).to(DEV), T, out, rms_weight=g, eps=1e-6, workspace=ws)
    torch.cuda.synchronize()
    for c0 in range(0, F, 4096):
        ref = oracle_mod.embed(codes[c0:c0 + 4096], T64, g64, 1e-6)
        compare_embed(out[c0:c0 + 4096].cpu().numpy(), ref, 1e-5)


def _prepared(T):
    P = torch.empty(dmel.dmel_table_prepare_size(T.shape[1], dmel.DMEL_BF16), dtype=torch.uint8, device=DEV)
    dmel.dmel_table_prepare(T, P)
    return P


@pytest.mark.parametrize("out_dt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("F", [1, 1000, 12288 + 77])
def test_embed_prepared_calls_match_oracle(F, out_dt, table_bf16, rmsw_bf16, oracle_mod):
    """With the table prepared once, calls of 12,288 frames or more take their RMSNorm scales from
    G (here a ragged last tile); smaller ones (one frame, one ragged tile) exchange row sums as
    unprepared calls do. Both match the oracle."""
    T, T64 = table_bf16
    g, g64 = rmsw_bf16
    P = _prepared(T)
    codes = synth.random_codes(45 + F, F)
    out = torch.empty((F, 6144), dtype=out_dt, device=DEV)
    ws = torch.empty(dmel.dmel_workspace_size(F, 6144, dmel.DMEL_BF16, True, True), dtype=torch.uint8, device=DEV)
    dmel.dmel_embed_prepared(torch.from_numpy(codes).to(DEV), T, out, P, rms_weight=g, eps=1e-6, workspace=ws)
    torch.cuda.synchronize()
    worst = 0.0
    for c0 in range(0, F, 4096):
        ref = oracle_mod.embed(codes[c0:c0 + 4096], T64, g64, 1e-6)
        got = out[c0:c0 + 4096].float().cpu().numpy()
        worst = max(worst, compare_embed(got, ref, 1e-5 if out_dt == torch.float32 else 1e-2))
    print(f"prepared embed F={F} out={out_dt}: worst {worst:.2e}")


def test_embed_prepared_equals_unprepared_at_gram_sizes(table_bf16, rmsw_bf16):
    """At 16,384 frames and more an unprepared call computes the same G itself: the outputs are
    bit-identical. Without RMSNorm the prepared data is ignored."""
    T, _ = table_bf16
    g, _ = rmsw_bf16
    P = _prepared(T)
    F = 16384 + 333
    codes = torch.from_numpy(synth.random_codes(46, F)).to(DEV)
    ws = torch.empty(dmel.dmel_workspace_size(F, 6144, dmel.DMEL_BF16, True, True), dtype=torch.uint8, device=DEV)
    a = torch.empty((F, 6144), dtype=torch.bfloat16, device=DEV)
    b = torch.empty_like(a)
    dmel.dmel_embed(codes, T, a, rms_weight=g, eps=1e-6, workspace=ws)
    dmel.dmel_embed_prepared(codes, T, b, P, rms_weight=g, eps=1e-6, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    dmel.dmel_embed(codes, T, a, workspace=ws)
    dmel.dmel_embed_prepared(codes, T, b, P, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_table_prepare_matches_the_gram_matrix(table_bf16):
    """The prepared data is G = T T^T as the Gram kernel writes it (bit-identical to the debug
    entry point's first block)."""
    T, _ = table_bf16
    P = _prepared(T)
    G = torch.full((2, 1280, 1280), float("nan"), dtype=torch.float32, device=DEV)
    dmel.dmel_debug_gram(T, G)
    torch.cuda.synchronize()
    got = P[:1280 * 1280 * 4].view(torch.float32).view(1280, 1280)
    for g in range(10):
        for h in range(g, 10):
            blk = (slice(128 * g, 128 * g + 128), slice(128 * h, 128 * h + 128))
            assert torch.equal(got[blk], G[0][blk]), (g, h)


def test_forward_prepared_batch64_10s(table_bf16, rmsw_bf16, oracle_mod):
    """FrontEnd(prepare=True): dmel_forward_prepared on the 64 x 10 s batch against the oracle."""
    T, T64 = table_bf16
    g, g64 = rmsw_bf16
    wav, off = synth.batch64_10s()
    fe = FrontEnd(T, g, 1e-6, torch.bfloat16, prepare=True)
    assert fe.prepared is not None
    plan = fe.plan(off)
    fe.forward(torch.from_numpy(wav).to(DEV), plan)
    torch.cuda.synchronize()
    _check_forward(wav, off, plan, T64, g64, 1e-2, oracle_mod, label="batch64_10s prepared")


# ------------------------------------------------------------- output rows (sentinel splice)

def _rows_case(F, S, seed):
    r = np.random.default_rng(seed)
    return r.choice(S, size=F, replace=False).astype(np.int64)


@pytest.mark.parametrize("out_dt", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rms", [True, False])
def test_embed_rows_scatter_into_sequence(out_dt, rms, table_bf16, rmsw_bf16, oracle_mod):
    """Frames written to arbitrary rows of a longer sequence: the mapped rows hold exactly what
    dmel_embed gives (same kernels, same arithmetic), within tolerance of the oracle; the other
    rows keep their contents."""
    T, T64 = table_bf16
    g, g64 = rmsw_bf16
    F, S = 700, 1000
    codes = synth.random_codes(61, F)
    cd = torch.from_numpy(codes).to(DEV)
    rows = _rows_case(F, S, 62)
    ws = torch.empty(max(dmel.dmel_workspace_size(F, 6144, dmel.DMEL_BF16, rms, True), 1), dtype=torch.uint8,
                     device=DEV)
    seq = torch.full((S, 6144), float("nan"), dtype=out_dt, device=DEV)
    dmel.dmel_embed_rows(cd, T, seq, torch.from_numpy(rows).to(DEV), rms_weight=g if rms else None, eps=1e-6,
                         workspace=ws)
    plain = torch.empty((F, 6144), dtype=out_dt, device=DEV)
    dmel.dmel_embed(cd, T, plain, rms_weight=g if rms else None, eps=1e-6, workspace=ws)
    torch.cuda.synchronize()
    got = seq.float().cpu().numpy()
    np.testing.assert_array_equal(got[rows], plain.float().cpu().numpy())
    ref = oracle_mod.embed(codes, T64, g64 if rms else None, 1e-6)
    compare_embed(got[rows], ref, 1e-5 if out_dt == torch.float32 else 1e-2)
    assert np.isnan(got[np.setdiff1d(np.arange(S), rows)]).all()
    assert dmel.dmel_get_device_error(clear=True) == 0


def test_embed_rows_fp32_table_cuda_cores(oracle_mod):
    T = synth.table(seed=9, dim=512)
    gw = synth.rms_weight(seed=10, dim=512)
    F, S = 77, 200
    codes = synth.random_codes(63, F)
    rows = _rows_case(F, S, 64)
    seq = torch.full((S, 512), float("nan"), dtype=torch.float32, device=DEV)
    dmel.dmel_embed_rows(torch.from_numpy(codes).to(DEV), torch.from_numpy(T).to(DEV), seq,
                         torch.from_numpy(rows).to(DEV), rms_weight=torch.from_numpy(gw).to(DEV), eps=1e-6)
    torch.cuda.synchronize()
    got = seq.cpu().numpy()
    compare_embed(got[rows], oracle_mod.embed(codes, T.astype(np.float64), gw.astype(np.float64), 1e-6), 1e-5)
    assert np.isnan(got[np.setdiff1d(np.arange(S), rows)]).all()


def test_embed_rows_out_of_range_rows_are_flagged_not_written(table_bf16, rmsw_bf16):
    T, _ = table_bf16
    g, _ = rmsw_bf16
    F, S = 300, 400
    rows = _rows_case(F, S, 65)
    rows[5], rows[200] = S, -1  # one past the end, negative
    codes = torch.from_numpy(synth.random_codes(66, F)).to(DEV)
    buf = torch.full((S + 8, 6144), float("nan"), dtype=torch.bfloat16, device=DEV)  # 8 guard rows past S
    ws = torch.empty(dmel.dmel_workspace_size(F, 6144, dmel.DMEL_BF16, True, True), dtype=torch.uint8, device=DEV)
    dmel.dmel_get_device_error(clear=True)
    dmel.dmel_embed_rows(codes, T, buf[:S], torch.from_numpy(rows).to(DEV), rms_weight=g, eps=1e-6, workspace=ws)
    torch.cuda.synchronize()
    assert dmel.dmel_get_device_error(clear=True) & dmel.DMEL_DEVERR_OUT_ROW
    got = buf.float().cpu().numpy()
    assert np.isnan(got[S:]).all()  # nothing past the sequence
    ok = np.delete(rows, [5, 200])
    assert np.isfinite(got[ok]).all()
    assert np.isnan(got[np.setdiff1d(np.arange(S), ok)]).all()


def test_forward_rows_splices_clips_at_their_sentinels(table_bf16, rmsw_bf16, oracle_mod):
    """Waveforms to the decoder's input sequence in one call: the planned rows hold the frames of
    dmel_forward, text rows keep the text embeddings, and the plan matches the oracle's
    expansion."""
    T, _ = table_bf16
    g, _ = rmsw_bf16
    wav, off = synth.batch64_10s()
    n_clips = 6
    lens = [160000, 32000, 700, 160000, 48000, 16000]  # the third clip is too short for a frame
    so = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    w = np.concatenate([wav[off[i]:off[i] + lens[i]] for i in range(n_clips)]).astype(np.float32)
    fo = dmel.dmel_frame_offsets(so)
    F = int(fo[-1])
    seq_len = 40
    sentinels = [2, 9, 10, 21, 30, 39]
    token_pos, frame_rows, S, audio = dmel.dmel_splice_plan(sentinels, fo, seq_len)
    otp, ofr, on, oa = oracle_mod.splice_plan(seq_len, sentinels, np.diff(fo).tolist())
    assert token_pos.tolist() == otp and frame_rows.tolist() == ofr and S == on and audio == oa == F
    seq = torch.full((S, 6144), 7.0, dtype=torch.bfloat16, device=DEV)  # stands for the text embeddings
    wd = torch.from_numpy(w).to(DEV)
    sod, fod = torch.from_numpy(so).to(DEV), torch.from_numpy(fo).to(DEV)
    ws = torch.empty(dmel.dmel_workspace_size(F, 6144, dmel.DMEL_BF16, True, False), dtype=torch.uint8, device=DEV)
    dmel.dmel_forward_rows(wd, sod, fod, F, T, seq, torch.from_numpy(frame_rows).to(DEV), rms_weight=g, eps=1e-6,
                           workspace=ws)
    ref = torch.empty((F, 6144), dtype=torch.bfloat16, device=DEV)
    dmel.dmel_forward(wd, sod, fod, F, T, ref, rms_weight=g, eps=1e-6, workspace=ws)
    torch.cuda.synchronize()
    got = seq.float().cpu().numpy()
    np.testing.assert_array_equal(got[frame_rows], ref.float().cpu().numpy())
    text = token_pos[token_pos >= 0]
    assert (got[text] == 7.0).all()
    assert dmel.dmel_get_device_error(clear=True) == 0


def test_embed_fp32_table_rmsnorm(oracle_mod):
    T = synth.table(seed=9, dim=512)
    gw = synth.rms_weight(seed=10, dim=512)
    F = 77
    codes = synth.random_codes(42, F)
    out = torch.empty((F, 512), dtype=torch.float32, device=DEV)
    dmel.dmel_embed(torch.from_numpy(codes).to(DEV), torch.from_numpy(T).to(DEV), out,
                    rms_weight=torch.from_numpy(gw).to(DEV), eps=1e-6)
    torch.cuda.synchronize()
    ref = oracle_mod.embed(codes, T.astype(np.float64), gw.astype(np.float64), 1e-6)
    compare_embed(out.cpu().numpy(), ref, 1e-5)


def test_embed_out_of_range_codes_are_flagged(table_bf16):
    T, _ = table_bf16
    codes = torch.zeros((130, 80), dtype=torch.uint8, device=DEV)
    codes[129, 5] = 200
    out = torch.empty((130, 6144), dtype=torch.bfloat16, device=DEV)
    dmel.dmel_embed(codes, T, out)
    assert dmel.dmel_get_device_error(clear=True) & dmel.DMEL_DEVERR_CODE_RANGE
    assert torch.isfinite(out.float()).all()


# ------------------------------------------------------------------------- full path, workloads

def _forward(wav, off, table, rmsw, out_dtype, tails=None):
    fe = FrontEnd(table, rmsw, 1e-6, out_dtype)
    plan = fe.plan(off)
    w = torch.from_numpy(wav).to(DEV)
    t_in = None if tails is None else torch.from_numpy(tails).to(DEV)
    fe.forward(w, plan, tails=t_in)
    torch.cuda.synchronize()
    return plan


def _check_forward(wav, off, plan, T64, g64, rtol, oracle_mod, frame_ids=None, embed_ids=None, label=""):
    gc = plan.codes.cpu().numpy()
    if frame_ids is None:
        oc, ol = oracle_mod.codes(wav, off)
        gsel = gc
    else:
        oc, ol = oracle_mod.codes(wav, off, frame_ids=frame_ids)
        gsel = gc[frame_ids]
    flips, flipped = compare_codes(gsel, oc, ol)
    ids = np.arange(gsel.shape[0]) if embed_ids is None else embed_ids
    ids = ids[~flipped[ids]]
    rows = ids if frame_ids is None else frame_ids[ids]
    worst = 0.0
    for c0 in range(0, len(ids), 2048):  # the fp64 oracle vectors, 2048 frames at a time
        ref = oracle_mod.embed(oc[ids[c0:c0 + 2048]], T64, g64, 1e-6)
        got = plan.out[torch.from_numpy(rows[c0:c0 + 2048]).to(DEV)].float().cpu().numpy()
        worst = max(worst, compare_embed(got, ref, rtol))
    print(f"{label}: frames {plan.n_frames}, code cells checked {gsel.size}, flips {flips}, "
          f"embeddings checked {len(ids)}, worst {worst:.2e}")


def test_forward_one_clip_2s_fp32(oracle_mod):
    wav, off = synth.one_clip_2s()
    T = synth.table()
    plan = _forward(wav, off, torch.from_numpy(T).to(DEV), None, torch.float32)
    _check_forward(wav, off, plan, T.astype(np.float64), None, 1e-5, oracle_mod, label="one_clip_2s")


def test_forward_batch64_10s(table_bf16, rmsw_bf16, oracle_mod):
    """Every frame: codes against the oracle, and every frame's vector (bar the few with a code
    flip at a level boundary) against the oracle's vector of the oracle's codes."""
    T, T64 = table_bf16
    g, g64 = rmsw_bf16
    wav, off = synth.batch64_10s()
    plan = _forward(wav, off, T, g, torch.bfloat16)
    assert plan.n_frames == 12800
    _check_forward(wav, off, plan, T64, g64, 1e-2, oracle_mod, label="batch64_10s")


def test_forward_host_pipelined_equals_single_call(table_bf16, rmsw_bf16):
    """The host path (copies of chunk i + 1 and i - 1 overlapping the kernels of chunk i) gives
    the same vectors and codes, bit for bit, as one device-side call on the whole batch."""
    T, _ = table_bf16
    g, _ = rmsw_bf16
    wav, off = synth.ragged1024(n_clips=40)
    fe = FrontEnd(T, g, 1e-6, torch.bfloat16)
    one = fe.plan(off)
    fe.forward(torch.from_numpy(wav).to(DEV), one)
    for chunk in (97, 1000, 0):
        p = fe.plan(off, chunk_frames=chunk, host_path=True)
        out_h = torch.empty((p.n_frames, T.shape[1]), dtype=torch.bfloat16).pin_memory()
        codes_h = torch.empty((p.n_frames, 80), dtype=torch.uint8).pin_memory()
        fe.forward_host(torch.from_numpy(wav).pin_memory(), p, out_h, codes_h)
        torch.cuda.synchronize()
        assert torch.equal(out_h, one.out.cpu()), chunk
        assert torch.equal(codes_h, one.codes.cpu()), chunk


def test_forward_long_20min(table_bf16, rmsw_bf16, oracle_mod):
    """Every one of the 24,000 frames, codes and vectors, against the oracle."""
    T, T64 = table_bf16
    g, g64 = rmsw_bf16
    wav, off = synth.long_20min()
    plan = _forward(wav, off, T, g, torch.bfloat16)
    assert plan.n_frames == 24000
    _check_forward(wav, off, plan, T64, g64, 1e-2, oracle_mod, label="long_20min")


def test_forward_ragged1024(table_bf16, rmsw_bf16, oracle_mod):
    T, T64 = table_bf16
    g, g64 = rmsw_bf16
    wav, off = synth.ragged1024()
    plan = _forward(wav, off, T, g, torch.bfloat16)
    fo = plan.frame_offsets_host
    r = np.random.default_rng(53)
    clips = r.choice(1024, 24, replace=False)
    ids = [np.arange(fo[c], fo[c + 1]) for c in clips]
    rest = r.choice(plan.n_frames, int(0.01 * plan.n_frames), replace=False)
    frame_ids = np.unique(np.concatenate(ids + [rest, [0, plan.n_frames - 1]])).astype(np.int64)
    emb = np.sort(r.choice(frame_ids.shape[0], 768, replace=False))
    _check_forward(wav, off, plan, T64, g64, 1e-2, oracle_mod, frame_ids=frame_ids, embed_ids=emb,
                   label="ragged1024 (sampled)")


def test_streaming_two_tail_buffers_equal_in_place(table_bf16, rmsw_bf16):
    """Streaming calls that alternate two tail buffers (the codes kernel writes the tails) give
    the same codes, vectors and tails, bit for bit, as calls that update one buffer in place."""
    T, _ = table_bf16
    g, _ = rmsw_bf16
    S = synth.Streams4096()
    fe = FrontEnd(T, g, 1e-6, torch.bfloat16)
    pa, pb = fe.plan(synth.offsets_from_lengths([800] * S.n)), fe.plan(synth.offsets_from_lengths([800] * S.n))
    t_in_place = torch.zeros((S.n, 800), device=DEV)
    bufs = [torch.zeros((S.n, 800), device=DEV), torch.zeros((S.n, 800), device=DEV)]
    for k in range(6):
        x = torch.from_numpy(S.call(k)).to(DEV).reshape(-1)
        fe.forward(x, pa, tails=t_in_place, tails_out=t_in_place)
        fe.forward(x, pb, tails=bufs[k % 2], tails_out=bufs[(k + 1) % 2])
        torch.cuda.synchronize()
        assert torch.equal(pa.codes, pb.codes) and torch.equal(pa.out, pb.out)
        assert torch.equal(t_in_place, bufs[(k + 1) % 2])


def test_streaming_4096_matches_offline_and_oracle(table_bf16, rmsw_bf16, oracle_mod):
    """4096 streams, 800 new samples per call plus the carried tail. Every call's codes and
    vectors equal those of one offline call on the concatenated stream (bit for bit), and
    sampled calls match the oracle."""
    T, T64 = table_bf16
    g, g64 = rmsw_bf16
    S = synth.Streams4096()
    n_calls = 1000
    check_calls = {0, 1, 2, 500, 999}
    fe = FrontEnd(T, g, 1e-6, torch.bfloat16)
    plan = fe.plan(synth.offsets_from_lengths([800] * S.n))
    tails = torch.zeros((S.n, 800), device=DEV)
    prev = None
    offline_streams = np.arange(0, S.n, 512)
    offline_wav = [[] for _ in offline_streams]
    offline_out = [[] for _ in offline_streams]
    for k in range(n_calls):
        x = S.call(k)
        for i, s in enumerate(offline_streams):
            if k < 40:
                offline_wav[i].append(x[s])
        fe.forward(torch.from_numpy(x).to(DEV).reshape(-1), plan, tails=tails, tails_out=tails)
        if k < 40:
            o = plan.out[torch.from_numpy(offline_streams).to(DEV)].cpu()
            for i in range(len(offline_streams)):
                offline_out[i].append(o[i])
        if k in check_calls:
            torch.cuda.synchronize()
            tail_in = prev if prev is not None else np.zeros((S.n, 800), np.float32)
            oc, ol = oracle_mod.codes(x.reshape(-1), plan.sample_offsets_host, tails=tail_in)
            flips, flipped = compare_codes(plan.codes.cpu().numpy(), oc, ol)
            ids = np.arange(0, S.n, 37)
            ids = ids[~flipped[ids]]
            ref = oracle_mod.embed(oc[ids], T64, g64, 1e-6)
            worst = compare_embed(plan.out[torch.from_numpy(ids).to(DEV)].float().cpu().numpy(), ref, 1e-2)
            print(f"stream call {k}: flips {flips}, worst {worst:.2e}")
        prev = x
    torch.cuda.synchronize()
    # streaming equals offline: 40 calls of selected streams against one call on their samples
    fe2 = FrontEnd(T, g, 1e-6, torch.bfloat16)
    for i in range(len(offline_streams)):
        wav = np.concatenate(offline_wav[i])
        p2 = fe2.plan(np.array([0, wav.size]))
        fe2.forward(torch.from_numpy(wav).to(DEV), p2)
        torch.cuda.synchronize()
        got = torch.stack(offline_out[i]).to(DEV)
        assert torch.equal(got, p2.out), f"stream {offline_streams[i]}: streaming differs from offline"
