"""The hMLP patchifier on the GPU against the oracle (vision path: "Inside Inkling: Audio
Design", Part 1 · Modeling, a 4-layer hMLP over 40x40 patches). The oracle sums in fp64 and rounds
to bf16 where the library stores bf16; the rule is the embeddings' (|y - o| <= rtol max(|o_j|,
rms(o))) with rtol 2e-2: an intermediate value that lands on the other side of a bf16 rounding
tie moves the next stage by a bf16 ulp (2^-8), which the later stages spread."""
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
    yield


def _params(seed, d1, d2, d3, D):
    r = np.random.default_rng(seed)
    p = {"W1": r.standard_normal((75, d1)) / np.sqrt(75), "b1": 0.1 * r.standard_normal(d1),
         "g1": 1 + 0.1 * r.standard_normal(d1), "be1": 0.1 * r.standard_normal(d1),
         "W2": r.standard_normal((4 * d1, d2)) / np.sqrt(4 * d1), "b2": 0.1 * r.standard_normal(d2),
         "g2": 1 + 0.1 * r.standard_normal(d2), "be2": 0.1 * r.standard_normal(d2),
         "W3": r.standard_normal((4 * d2, d3)) / np.sqrt(4 * d2), "b3": 0.1 * r.standard_normal(d3),
         "g3": 1 + 0.1 * r.standard_normal(d3), "be3": 0.1 * r.standard_normal(d3),
         "W4": r.standard_normal((4 * d3, D)) / np.sqrt(4 * d3), "b4": 0.1 * r.standard_normal(D)}
    dev, host = {}, {}
    for k, v in p.items():
        if k.startswith("W"):
            t = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)
            dev[k], host[k] = t.to(DEV).contiguous(), t.double().numpy()
        else:
            t = torch.from_numpy(v.astype(np.float32))
            dev[k], host[k] = t.to(DEV).contiguous(), t.double().numpy()
    return dev, host


def _images(seed, n, H, W):
    r = np.random.default_rng(seed)
    t = torch.from_numpy(r.uniform(-1, 1, (n, H, W, 3)).astype(np.float32)).to(torch.bfloat16)
    return t.to(DEV).contiguous(), t.double().numpy()


@pytest.mark.parametrize("widths", [(16, 24, 32, 40), (1536, 1536, 1536, 6144)])
def test_hmlp_matches_oracle(widths, oracle_mod):
    dev, host = _params(90, *widths)
    img_d, img_h = _images(91, 2, 80, 120)  # 2 images of 2 x 3 patches
    P = 12
    out = torch.empty((P, widths[3]), dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(dmel.dmel_hmlp_workspace_size(P, dev), dtype=torch.uint8, device=DEV)
    dmel.dmel_hmlp(img_d, dev, out, ws)
    torch.cuda.synchronize()
    ref = oracle_mod.hmlp(img_h, host)
    worst = compare_embed(out.float().cpu().numpy(), ref, 2e-2)
    print(f"hmlp widths {widths}: worst {worst:.2e}")


def test_hmlp_patch_order_and_no_patches():
    dev, _ = _params(92, 8, 8, 8, 16)
    img_d, _ = _images(93, 1, 40, 80)
    ws = torch.empty(dmel.dmel_hmlp_workspace_size(4, dev), dtype=torch.uint8, device=DEV)
    a = torch.empty((2, 16), dtype=torch.bfloat16, device=DEV)
    b = torch.empty((2, 16), dtype=torch.bfloat16, device=DEV)
    dmel.dmel_hmlp(img_d, dev, a, ws)
    dmel.dmel_hmlp(torch.cat([img_d[:, :, 40:], img_d[:, :, :40]], dim=2).contiguous(), dev, b, ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b.flip(0))  # patches are independent and come out in raster order
    empty = torch.empty((0, 40, 40, 3), dtype=torch.bfloat16, device=DEV)
    dmel.dmel_hmlp(empty, dev, a, ws)  # no image: a no-op
