"""Host logic of dmel_forward_host: the chunk plan must give every frame of the batch exactly the
1600 samples the causal framing assigns it ("Inside Inkling: Audio Design", Part 1 · Modeling:
hop 800, window 1600; samples before a clip are zero), whatever the chunk size, with chunks cut
inside clips, clips too short for a frame, and one-frame clips. Runs on the CPU: the plan is pure
host code, checked here by rebuilding each frame's window from what the plan copies."""
import numpy as np
import pytest

from encoder_free_audio_b200 import build, dmel, synth


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def _windows_from_plan(so_global, chunk_frames):
    """Each frame's window, as sample indices of the batch (-1 = zero), rebuilt from the plan:
    the copied range [s_lo, s_hi), the first piece's tail, zero tails for the other pieces."""
    plan = dmel.dmel_debug_forward_host_plan(so_global, chunk_frames)
    wins = []
    prev_f1 = 0
    for ch in plan:
        assert ch["f0"] == prev_f1 and ch["f1"] > ch["f0"]
        assert ch["f1"] - ch["f0"] <= chunk_frames
        prev_f1 = ch["f1"]
        base = ch["s_lo"] + (800 if ch["tail"] else 0)  # first piece's first sample
        so, fo = ch["so"], ch["fo"]
        n = so.shape[0] - 1
        assert fo[0] == 0 and fo[-1] == ch["f1"] - ch["f0"] and so[0] == 0 and so[-1] == ch["s_hi"] - base
        assert np.all(np.diff(fo) >= 1), "every piece has a frame"
        for p in range(n):
            length = so[p + 1] - so[p]
            for t in range(fo[p + 1] - fo[p]):
                assert 800 * (t + 1) <= length, "a piece's frames lie inside its samples"
                idx = np.arange(800 * (t - 1), 800 * (t + 1))
                w = base + so[p] + idx
                if t == 0:
                    tail = (np.arange(ch["s_lo"], ch["s_lo"] + 800) if (p == 0 and ch["tail"])
                            else np.full(800, -1))
                    w[:800] = tail
                wins.append(w)
    return np.array(wins), prev_f1


def _windows_direct(so):
    wins = []
    for c in range(so.shape[0] - 1):
        for t in range((so[c + 1] - so[c]) // 800):
            idx = np.arange(800 * (t - 1), 800 * (t + 1))
            wins.append(np.where(idx >= 0, so[c] + idx, -1))
    return np.array(wins)


@pytest.mark.parametrize("chunk_frames", [1, 3, 7, 64, 1000, 8192])
def test_plan_gives_every_frame_its_window(chunk_frames):
    rng = np.random.default_rng(5)
    # lengths: no frame (0, 1, 799), exactly one frame (800, 1599), ragged and long clips
    lengths = [0, 799, 800, 1599, 1600, 33_333, 1, 12_000, 800 * 37 + 5] + list(rng.integers(0, 40_000, 20))
    so = synth.offsets_from_lengths(lengths)
    got, F = _windows_from_plan(so, chunk_frames)
    ref = _windows_direct(so)
    assert F == ref.shape[0] == got.shape[0]
    assert np.array_equal(got, ref)


def test_plan_of_one_long_clip_cuts_inside_it():
    so = synth.offsets_from_lengths([19_200_000])  # 20 minutes: 24,000 frames
    plan = dmel.dmel_debug_forward_host_plan(so, 8192)
    assert [(c["f0"], c["f1"], c["tail"]) for c in plan] == [(0, 8192, False), (8192, 16384, True),
                                                            (16384, 24000, True)]
    # a chunk that starts inside the clip copies the 800 samples before its first frame's hop
    assert plan[1]["s_lo"] == 800 * (8192 - 1) and plan[1]["s_hi"] == 800 * 16384


def test_workspace_size_and_plan_reject_bad_offsets():
    assert dmel.dmel_forward_host_workspace_size([0, 10, 5], 6144, dmel.DMEL_BF16, dmel.DMEL_BF16, True) == 0
    assert dmel.dmel_forward_host_workspace_size([3, 10], 6144, dmel.DMEL_BF16, dmel.DMEL_BF16, True) == 0
    assert dmel.dmel_forward_host_workspace_size([0, 799], 6144, dmel.DMEL_BF16, dmel.DMEL_BF16, True) == 0
    assert dmel.dmel_forward_host_workspace_size([0, 800], 6144, dmel.DMEL_BF16, dmel.DMEL_BF16, True) > 0
    with pytest.raises(dmel.DmelError):
        dmel.dmel_debug_forward_host_plan([0, 1600], 0)
    with pytest.raises(dmel.DmelError):
        dmel.dmel_debug_forward_host_plan([0, 1600, 800], 4)
