"""dmel_forward_host (host waveforms in, host vectors out, copies overlapped with the kernels,
chunks cut inside clips) against dmel_forward on device buffers and against the oracle at the
frames right after each cut (they take their first 800 samples from the chunk's tail)."""
import numpy as np
import pytest
import torch

from encoder_free_audio_b200 import build, dmel, synth
from helpers import bf16_table, compare_codes, compare_embed

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    dmel.dmel_get_device_error(clear=True)
    yield
    assert dmel.dmel_get_device_error(clear=True) == 0


def _device_forward(wav, off, T, G, out_dtype):
    fo = dmel.dmel_frame_offsets(off)
    F = int(fo[-1])
    out = torch.empty((F, T.shape[1]), dtype=out_dtype, device=DEV)
    codes = torch.empty((F, 80), dtype=torch.uint8, device=DEV)
    ws_n = dmel.dmel_workspace_size(F, T.shape[1], dmel._dtype_code(T), G is not None, True)
    ws = torch.empty(max(1, ws_n), dtype=torch.uint8, device=DEV)
    dmel.dmel_forward(torch.from_numpy(wav).to(DEV), torch.from_numpy(off).to(DEV), torch.from_numpy(fo).to(DEV), F,
                      T, out, rms_weight=G, eps=1e-6, codes_out=codes, workspace=ws)
    torch.cuda.synchronize()
    return out.cpu(), codes.cpu()


def _host_forward(wav, off, T, G, out_dtype, chunk_frames, pinned=True):
    F = int(dmel.dmel_frame_offsets(off)[-1])
    wav_h = torch.from_numpy(wav)
    out_h = torch.full((F, T.shape[1]), float("nan"), dtype=out_dtype)
    codes_h = torch.full((F, 80), 255, dtype=torch.uint8)
    if pinned:
        wav_h, out_h, codes_h = wav_h.pin_memory(), out_h.pin_memory(), codes_h.pin_memory()
    n = dmel.dmel_forward_host_workspace_size(off, T.shape[1], dmel._dtype_code(T), dmel._dtype_code(out_h),
                                              G is not None, chunk_frames)
    ws = torch.empty(max(1, n), dtype=torch.uint8, device=DEV)
    dmel.dmel_forward_host(wav_h, off, T, out_h, rms_weight=G, eps=1e-6, codes_host=codes_h,
                           chunk_frames=chunk_frames, workspace=ws)
    torch.cuda.current_stream().synchronize()
    return out_h, codes_h


def _cut_frames(off, chunk_frames):
    """The first frame of every chunk that starts inside a clip, and the frame after it."""
    ids = []
    for ch in dmel.dmel_debug_forward_host_plan(off, chunk_frames):
        if ch["tail"]:
            ids += [ch["f0"], ch["f0"] + 1]
    return np.array(sorted(set(i for i in ids)), np.int64)


def test_forward_host_batch64_matches_device_path_and_oracle(oracle_mod):
    wav, off = synth.batch64_10s()
    t, t64 = bf16_table(synth.table())
    T = t.to(DEV)
    g = torch.from_numpy(synth.rms_weight()).to(torch.bfloat16)
    G = g.to(DEV)
    ref_out, ref_codes = _device_forward(wav, off, T, G, torch.bfloat16)
    for chunk in (1000, 8192):  # 1000 cuts inside clips (200 frames each); 8192 the default size
        out_h, codes_h = _host_forward(wav, off, T, G, torch.bfloat16, chunk)
        assert torch.equal(codes_h, ref_codes)
        assert torch.equal(out_h, ref_out), f"chunk_frames {chunk}: host pipeline differs from dmel_forward"
    # frames right after the cuts, against the oracle
    ids = _cut_frames(off, 1000)
    ids = ids[ids < ref_codes.shape[0]]
    oc, ol = oracle_mod.codes(wav, off, frame_ids=ids)
    compare_codes(codes_h.numpy()[ids], oc, ol)
    ref = oracle_mod.embed(oc, t64, g.double().numpy(), 1e-6)
    compare_embed(out_h.float().numpy()[ids], ref, 1e-2)


def test_forward_host_ragged_fp32_small_chunks(oracle_mod):
    r = np.random.default_rng(31)
    lengths = [0, 1, 799, 800, 1599, 4000, 33_333, 800, 0, 12_345, 800 * 11 + 3]
    off = synth.offsets_from_lengths(lengths)
    wav = r.uniform(-0.8, 0.8, int(off[-1])).astype(np.float32)
    T = torch.from_numpy(synth.table(dim=512)).to(DEV)  # fp32 table: the CUDA-core embedding
    ref_out, ref_codes = _device_forward(wav, off, T, None, torch.float32)
    for chunk, pinned in ((7, True), (3, False), (1, True)):
        out_h, codes_h = _host_forward(wav, off, T, None, torch.float32, chunk, pinned=pinned)
        assert torch.equal(codes_h, ref_codes)
        assert torch.equal(out_h, ref_out), f"chunk_frames {chunk} pinned {pinned}"
    oc, ol = oracle_mod.codes(wav, off)
    compare_codes(codes_h.numpy(), oc, ol)
    compare_embed(out_h.numpy(), oracle_mod.embed(oc, synth.table(dim=512).astype(np.float64)), 1e-5)


def test_forward_host_rejects_a_small_workspace():
    off = synth.offsets_from_lengths([16_000])
    wav = torch.zeros(16_000)
    T = torch.zeros((1280, 256), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((20, 256), dtype=torch.bfloat16)
    n = dmel.dmel_forward_host_workspace_size(off, 256, dmel.DMEL_BF16, dmel.DMEL_BF16, False, 0)
    ws = torch.empty(n - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(dmel.DmelError):
        dmel.dmel_forward_host(wav, off, T, out, workspace=ws)
    # no frame: nothing to do, no workspace needed
    dmel.dmel_forward_host(torch.zeros(700), [0, 700], T, torch.empty((0, 256), dtype=torch.bfloat16))
