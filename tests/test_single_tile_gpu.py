"""The one-CTA tensor-core tiles (DMEL_EMBED_TILE=single) against the oracle: the embedding
parity tests run again in a fresh process with CTA pairs switched off, so both tile shapes of
the tcgen05 kernel stay covered."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_embedding_parity_with_single_cta_tiles():
    env = dict(os.environ, DMEL_EMBED_TILE="single")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_parity_gpu.py"), "-k", "embed or batch64"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
