"""The RMSNorm scales' arithmetic on the host: a frame's sum of squares taken from the table's
Gram matrix G = T T^T (in blocks of 8 x 8 bins, diagonal terms once and every other pair twice)
equals the sum of squares of the frame's summed rows ("Inside Inkling: Audio Design", Part 1 ·
Modeling: the 80 rows are summed, then an optional RMSNorm), for random codes and tables, for
codes that pick the same level everywhere and for the extreme levels."""
import numpy as np
import pytest

from encoder_free_audio_b200 import build, dmel, synth


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def _direct(T64, codes):
    rows = 16 * np.arange(80) + codes.astype(np.int64)
    x = T64[rows].sum(axis=0)
    return float(x @ x)


@pytest.mark.parametrize("dim", [64, 512, 6144])
def test_gram_sumsq_equals_direct_sum_of_squares(dim):
    r = np.random.default_rng(dim)
    T64 = r.normal(0.0, 0.02, (1280, dim))
    G = (T64 @ T64.T).astype(np.float32)
    cases = [r.integers(0, 16, 80).astype(np.uint8) for _ in range(20)]
    cases += [np.zeros(80, np.uint8), np.full(80, 15, np.uint8), (np.arange(80) % 16).astype(np.uint8)]
    for c in cases:
        got = dmel.dmel_debug_norm_sumsq_host(c, G)
        ref = _direct(T64, c)
        # fp32 G entries and fp32 sums of 3,240 terms: a few 1e-7 of the sum at most
        assert abs(got - ref) <= 2e-6 * ref, (got, ref)


def test_gram_sumsq_uses_each_pair_with_its_weight():
    """An integer table, so every G entry and every partial sum is exact in fp32: the result must
    equal the direct sum bit for bit (a dropped pair, a pair counted once, a transposed block or a
    wrong diagonal weight all change it)."""
    r = np.random.default_rng(3)
    T = r.integers(-3, 4, (1280, 40)).astype(np.float64)
    G = (T @ T.T).astype(np.float32)
    for seed in range(10):
        c = np.random.default_rng(seed).integers(0, 16, 80).astype(np.uint8)
        assert dmel.dmel_debug_norm_sumsq_host(c, G) == _direct(T, c)
    # a G whose upper blocks only hold the truth: the lower blocks are never read
    c = synth.random_codes(5, 1)[0]
    Gu = G.copy()
    for g in range(10):
        for h in range(g):
            Gu[128 * g:128 * g + 128, 128 * h:128 * h + 128] = np.nan
    assert dmel.dmel_debug_norm_sumsq_host(c, Gu) == _direct(T, c)
