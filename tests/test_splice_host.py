"""The library's host splice plan (dmel_splice_plan) against the oracle's plain expansion
("Inside Inkling: Audio Design", Part 3 · Inference: one sentinel per audio item expands into
its frames), and its argument checks. No GPU."""
import json
import os

import numpy as np
import pytest

from encoder_free_audio_b200 import dmel

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "splice_example.json")


def _fo(frames):
    return np.concatenate([[0], np.cumsum(frames)]).astype(np.int64)


def test_golden_example():
    g = json.load(open(GOLDEN))
    tp, fr, n, a = dmel.dmel_splice_plan(g["sentinel_pos"], _fo(g["frames_per_item"]), g["seq_len"])
    assert tp.tolist() == g["token_pos"] and fr.tolist() == g["frame_rows"]
    assert n == g["expanded_len"] and a == g["audio_tokens"]


@pytest.mark.parametrize("seed", range(20))
def test_matches_oracle(oracle_mod, seed):
    r = np.random.default_rng(700 + seed)
    seq_len = int(r.integers(1, 400))
    k = int(r.integers(0, min(seq_len, 40) + 1))
    pos = sorted(r.choice(seq_len, size=k, replace=False).tolist())
    f = r.integers(0, 600, size=k).tolist()  # up to 30 s per clip
    tp, fr, n, a = dmel.dmel_splice_plan(pos, _fo(f), seq_len)
    otp, ofr, on, oa = oracle_mod.splice_plan(seq_len, pos, f)
    assert tp.tolist() == otp and fr.tolist() == ofr and n == on and a == oa


def test_frame_counts_from_clip_lengths():
    # the plan takes the frame offsets dmel_frame_offsets gives for the clips' sample counts
    so = np.array([0, 32000, 32000 + 799, 32000 + 799 + 160000], np.int64)
    fo = dmel.dmel_frame_offsets(so)
    assert fo.tolist() == [0, 40, 40, 240]
    tp, fr, n, a = dmel.dmel_splice_plan([0, 5, 9], fo, 10)
    assert a == 240 and n == 10 + 39 - 1 + 199
    assert fr[:40].tolist() == list(range(40)) and fr[40:].tolist() == list(range(9 + 38, 9 + 38 + 200))


@pytest.mark.parametrize("pos,fo,seq_len", [
    ([3, 3], [0, 1, 2], 5),      # not strictly increasing
    ([2, 1], [0, 1, 2], 5),
    ([5], [0, 1], 5),            # outside the sequence
    ([-1], [0, 1], 5),
    ([1], [1, 2], 5),            # frame offsets not starting at 0
    ([1, 2], [0, 3, 2], 5),      # decreasing frame offsets
])
def test_rejects_bad_plans(pos, fo, seq_len):
    with pytest.raises(dmel.DmelError):
        dmel.dmel_splice_plan(pos, fo, seq_len)


@pytest.mark.parametrize("seq_len,pos,f", [
    (0, [], []),                        # empty sequence, no audio
    (4, [], []),                        # text only: identity
    (3, [0, 1, 2], [2, 0, 3]),          # every position a sentinel, one clip without frames
    (5, [0, 4], [1, 1]),                # one-frame clips at both ends: the length is unchanged
    (6, [5], [0]),                      # a frameless clip at the end drops the last position
    (2, [0], [100000]),                 # one long clip
])
def test_edge_cases_match_oracle(oracle_mod, seq_len, pos, f):
    tp, fr, n, a = dmel.dmel_splice_plan(pos, _fo(f), seq_len)
    otp, ofr, on, oa = oracle_mod.splice_plan(seq_len, pos, f)
    assert tp.tolist() == otp and fr.tolist() == ofr and n == on and a == oa
    # every expanded position is filled exactly once, by a text token or by a frame
    filled = sorted([p for p in tp.tolist() if p >= 0] + fr.tolist())
    assert filled == list(range(n))
