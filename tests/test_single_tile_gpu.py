"""The other tensor-core kernels against the oracle: the embedding parity tests run again in a
fresh process with the RMSNorm scales taken from the table's Gram matrix at every call size
(DMEL_EMBED_NORM=gram; by default only calls of 16,384 frames or more do), with the resident-table
kernel switched on (DMEL_EMBED_TABLE=resident: each CTA
pair keeps its column slice of the table in shared memory), with the 2:4-sparse product switched
off (DMEL_EMBED_MMA=dense: dense CTA-pair tiles) and with CTA pairs switched off
(DMEL_EMBED_TILE=single: dense one-CTA tiles), so every tile shape of the tcgen05 path stays
covered."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_embed_parity(**env_overrides):
    env = dict(os.environ, **env_overrides)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_parity_gpu.py"), "-k", "embed or batch64"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


def test_embedding_parity_with_gram_norm_at_every_size():
    _run_embed_parity(DMEL_EMBED_NORM="gram")


def test_embedding_parity_with_resident_table_slices():
    _run_embed_parity(DMEL_EMBED_TABLE="resident")


def test_embedding_parity_with_dense_pair_tiles():
    _run_embed_parity(DMEL_EMBED_MMA="dense")


def test_embedding_parity_with_single_cta_tiles():
    _run_embed_parity(DMEL_EMBED_TILE="single")
