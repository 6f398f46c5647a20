"""ShortConv on the GPU against the oracle ("Inside Inkling: Audio Design", Part 3 · Inference:
y = x + sum_{d<4} w_d x_{t-d} per channel, per sequence, with a carried per-request state)."""
import numpy as np
import pytest
import torch

from encoder_free_audio_b200 import build, dmel
from helpers import compare_embed

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    dmel.library()
    dmel.dmel_get_device_error(clear=True)
    yield


def _case(seed, lens, C, dt):
    r = np.random.default_rng(seed)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    x = r.standard_normal((int(off[-1]), C)).astype(np.float32)
    w = (0.5 * r.standard_normal((C, 4))).astype(np.float32)
    st = r.standard_normal((len(lens), 3, C)).astype(np.float32)
    if dt == torch.bfloat16:  # the oracle sees exactly the bf16 values the kernel reads
        x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
        st = torch.from_numpy(st).to(torch.bfloat16).float().numpy()
    return off, x, w, st


def _run(off, x, w, st, dt, with_state=True, want_state=True):
    xd = torch.from_numpy(x).to(dt).to(DEV)
    y = torch.empty_like(xd)
    sd = torch.from_numpy(st).to(dt).to(DEV) if with_state else None
    so = torch.full((off.shape[0] - 1, 3, x.shape[1]), 9.0, dtype=dt, device=DEV) if want_state else None
    dmel.dmel_shortconv(xd, torch.from_numpy(off).to(DEV), torch.from_numpy(w).to(DEV), y, state=sd, state_out=so)
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), (None if so is None else so.float().cpu().numpy())


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("with_state", [True, False])
def test_shortconv_ragged_matches_oracle(dt, with_state, oracle_mod):
    # sequences of 0..3 tokens (the carried state reaches into the output), runs that straddle
    # sequence starts, and a long one
    lens = [0, 1, 2, 3, 4, 0, 31, 32, 33, 7, 500, 1, 0]
    C = 264
    off, x, w, st = _case(81, lens, C, dt)
    y, so = _run(off, x, w, st, dt, with_state=with_state)
    ry, rso = oracle_mod.shortconv(x, off, w, st if with_state else None)
    compare_embed(y, ry, 1e-5 if dt == torch.float32 else 1e-2)
    np.testing.assert_array_equal(so, rso.astype(np.float32))  # state rows are copies of inputs
    assert dmel.dmel_get_device_error(clear=True) == 0


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_shortconv_channel_slices_and_long_runs(dt, oracle_mod):
    """2056 channels (a full 2048-channel slice and one of 8), sequences long enough that each
    block's run of tokens starts inside a sequence and crosses into the next one."""
    lens = [0, 2, 900, 1, 1500, 3, 0, 777]
    C = 2056
    off, x, w, st = _case(84, lens, C, dt)
    for with_state in (True, False):
        y, so = _run(off, x, w, st, dt, with_state=with_state)
        ry, rso = oracle_mod.shortconv(x, off, w, st if with_state else None)
        compare_embed(y, ry, 1e-5 if dt == torch.float32 else 1e-2)
        np.testing.assert_array_equal(so, rso.astype(np.float32))
    assert dmel.dmel_get_device_error(clear=True) == 0


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_shortconv_decode_token_by_token_equals_offline(dt):
    """Serving: one call per decode step with the state updated in place gives, bit for bit,
    what one call over the whole sequences gives."""
    lens = [40, 17, 64]
    C = 128
    off, x, w, _ = _case(82, lens, C, dt)
    y_all, s_all = _run(off, x, w, np.zeros((3, 3, C), np.float32), dt, with_state=False)
    xd = torch.from_numpy(x).to(dt).to(DEV)
    wd = torch.from_numpy(w).to(DEV)
    state = torch.zeros((3, 3, C), dtype=dt, device=DEV)
    y_steps = torch.empty_like(xd)
    for t in range(max(lens)):
        # step t: one token from every sequence that still has one (a batch of decode requests)
        alive = [s for s in range(3) if t < lens[s]]
        rows = torch.tensor([off[s] + t for s in alive], device=DEV)
        xs = xd[rows].contiguous()
        ys = torch.empty_like(xs)
        st = state[alive].contiguous()
        dmel.dmel_shortconv(xs, torch.arange(len(alive) + 1, dtype=torch.int64, device=DEV), wd, ys, state=st,
                            state_out=st)
        state[alive] = st
        y_steps[rows] = ys
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y_steps.float().cpu().numpy(), y_all)
    np.testing.assert_array_equal(state.float().cpu().numpy(), s_all)


def test_shortconv_model_width(oracle_mod):
    """6144 channels, 12,800 tokens in 64 sequences of 200 (the batch workload's frame count),
    bf16: every output against the oracle."""
    lens = [200] * 64
    off, x, w, st = _case(83, lens, 6144, torch.bfloat16)
    y, so = _run(off, x, w, st, torch.bfloat16)
    ry, rso = oracle_mod.shortconv(x, off, w, st)
    compare_embed(y, ry, 1e-2)
    np.testing.assert_array_equal(so, rso.astype(np.float32))


def test_shortconv_bad_offsets_are_flagged():
    C = 16
    x = torch.zeros((10, C), device=DEV)
    y = torch.empty_like(x)
    w = torch.zeros((C, 4), device=DEV)
    off = torch.tensor([0, 12], dtype=torch.int64, device=DEV)  # says 12 tokens, x holds 10
    so = torch.empty((1, 3, C), device=DEV)
    dmel.dmel_get_device_error(clear=True)
    dmel.dmel_shortconv(x, off, w, y, state_out=so)
    torch.cuda.synchronize()
    assert dmel.dmel_get_device_error(clear=True) & dmel.DMEL_DEVERR_OFFSETS
