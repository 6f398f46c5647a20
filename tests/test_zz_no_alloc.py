"""dmel_embed_noalloc: the embedding for callers that cannot allocate device memory (a real-time
audio callback, a step being captured into a CUDA graph, a host framework that owns all device
memory). It must give what dmel_embed gives with a caller workspace, call after call, while the
partial sums live in the library's fixed scratch array. Collected last on purpose, so a failure
here comes after every other test has run."""
import ctypes

import numpy as np
import pytest
import torch

from encoder_free_audio_b200 import build, dmel, synth
from helpers import bf16_table, compare_embed

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    return dmel.library()


def _call_noalloc(lib, codes, table, out, g, eps=1e-6):
    """The C entry point itself, through ctypes, on the current stream."""
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    out_code = dmel.DMEL_BF16 if out.dtype == torch.bfloat16 else dmel.DMEL_F32
    return lib.dmel_embed_noalloc(ctypes.c_void_p(codes.data_ptr()), codes.shape[0], ctypes.c_void_p(table.data_ptr()),
                                  dmel.DMEL_BF16, table.shape[1],
                                  None if g is None else ctypes.c_void_p(g.data_ptr()), ctypes.c_float(eps),
                                  ctypes.c_void_p(out.data_ptr()), out_code, stream)


def test_noalloc_matches_workspace_entry_point_twice(lib, oracle_mod):
    t_cpu, t64 = bf16_table(synth.table())
    T = t_cpu.to(DEV)
    g_cpu = torch.from_numpy(synth.rms_weight()).to(torch.bfloat16)
    g = g_cpu.to(DEV)
    dmel.dmel_get_device_error(clear=True)
    # calls in a row against dmel_embed with its own workspace: same kernel, same arithmetic, so
    # the vectors must be identical bit for bit. The frame counts grow, so a later call reads
    # scratch the earlier ones never wrote; the last call writes fp32.
    for call, (F, out_dtype) in enumerate(((777, torch.bfloat16), (2000, torch.bfloat16), (4321, torch.float32))):
        codes = torch.from_numpy(synth.random_codes(100 + call, F)).to(DEV)
        out_na = torch.empty((F, 6144), dtype=out_dtype, device=DEV)
        assert _call_noalloc(lib, codes, T, out_na, g) == dmel.DMEL_OK
        out_ws = torch.empty_like(out_na)
        ws = torch.empty(dmel.dmel_workspace_size(F, 6144, dmel.DMEL_BF16, True, True), dtype=torch.uint8,
                         device=DEV)
        dmel.dmel_embed(codes, T, out_ws, rms_weight=g, eps=1e-6, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(out_na, out_ws), f"call {call}: no-alloc output differs from dmel_embed"
    # and the last call against the oracle on a sample of its frames
    ids = np.arange(0, F, 97)
    ref = oracle_mod.embed(codes.cpu().numpy()[ids], t64, g_cpu.double().numpy(), 1e-6)
    compare_embed(out_na.cpu().numpy()[ids], ref, 1e-5)
    assert dmel.dmel_get_device_error(clear=True) == 0


def test_noalloc_rejects_requests_beyond_its_scratch(lib):
    """The fixed scratch holds the row sums of squares the CTAs of a row exchange: 128-frame tiles
    x ceil(6144 / 192) = 32 column tiles x 128 floats, plus one counter per tile, which is 4 MiB
    or less up to 32,640 frames at width 6144 and more from 32,641 frames on."""
    T = torch.zeros((1280, 6144), dtype=torch.bfloat16, device=DEV)
    g = torch.ones(6144, dtype=torch.bfloat16, device=DEV)
    F = 32641
    codes = torch.zeros((F, 80), dtype=torch.uint8, device=DEV)
    out = torch.empty((F, 6144), dtype=torch.bfloat16, device=DEV)
    assert _call_noalloc(lib, codes, T, out, g) == dmel.DMEL_ERR_TOO_LARGE
    assert _call_noalloc(lib, codes[:32640], T, out[:32640], g) == dmel.DMEL_OK
    # without RMSNorm the request needs no scratch and runs
    assert _call_noalloc(lib, codes[:300], T, out[:300], None) == dmel.DMEL_OK
    torch.cuda.synchronize()
