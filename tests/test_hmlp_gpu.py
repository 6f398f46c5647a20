"""The hMLP patchifier on the GPU against the oracle (vision path: "Inside Inkling: Audio
Design", Part 1 · Modeling, a 4-layer hMLP over 40x40 patches). The oracle sums in fp64 and rounds
to bf16 where the library stores bf16; the rule is the embeddings' (|y - o| <= rtol max(|o_j|,
rms(o))) with rtol 2e-2: an intermediate value that lands on the other side of a bf16 rounding
tie moves the next stage by a bf16 ulp (2^-8), which the later stages spread."""
import math

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


def _patch_oracle(oracle_mod, img_h, host, p, H, W):
    """The oracle on patch p alone (patches are independent; raster order within an image)."""
    pw, ph = W // 40, H // 40
    i, pr, pc = p // (ph * pw), (p // pw) % ph, p % pw
    return oracle_mod.hmlp(img_h[i:i + 1, 40 * pr:40 * pr + 40, 40 * pc:40 * pc + 40], host)[0]


@pytest.mark.parametrize("widths,n,H,W", [
    ((256, 64, 64, 64), 1, 80, 240),              # one 256-column chunk per row, 12 patches
    ((512, 64, 64, 64), 1, 520, 920),             # 299 patches: 150 two-patch tiles, the last ragged
    ((1536, 1536, 1536, 6144), 4, 800, 800),      # the measured workload: 1,600 patches
])
def test_hmlp_fused_stage1_sampled(widths, n, H, W, oracle_mod):
    """The fused stage-1 kernel (d1 a multiple of 256): whole output at 12 patches, else patches
    sampled across the persistent schedule (first and last tiles, tiles past the first wave of
    blocks, the ragged last tile's single patch) against the oracle one patch at a time."""
    dev, host = _params(94 + widths[0], *widths)
    img_d, img_h = _images(95, n, H, W)
    P = n * (H // 40) * (W // 40)
    out = torch.empty((P, widths[3]), dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(dmel.dmel_hmlp_workspace_size(P, dev), dtype=torch.uint8, device=DEV)
    dmel.dmel_hmlp(img_d, dev, out, ws)
    torch.cuda.synchronize()
    assert dmel.dmel_get_device_error(clear=True) == 0
    got = out.float().cpu().numpy()
    if P <= 12:
        picks = list(range(P))
    else:
        r = np.random.default_rng(96)
        picks = sorted({0, 1, 2 * 147, 2 * 147 + 1, 2 * 148, 2 * 148 + 1, P - 2, P - 1,
                        *r.integers(0, P, 4).tolist()} & set(range(P)))
    ref = np.stack([_patch_oracle(oracle_mod, img_h, host, p, H, W) for p in picks])
    worst = compare_embed(got[picks], ref, 2e-2)
    print(f"hmlp fused widths {widths}, {P} patches, {len(picks)} checked: worst {worst:.2e}")


def test_gelu_formula_within_its_error_bound():
    """The kernels' GELU, u Phi(u) with erfc from Abramowitz & Stegun 7.1.26 (absolute error at
    most 1.5e-7, so at most 7.5e-8 in Phi), against the exact u Phi(u) in fp64 on a dense sweep,
    the tails and signed zeros: |y - GELU(u)| <= |u| (7.5e-8 + 4e-7 of fp32 rounding in the
    reciprocal, exp2 and polynomial) + one fp32 rounding of the result."""
    u = torch.cat([torch.linspace(-12.0, 12.0, (1 << 20) + 1, dtype=torch.float64),
                   torch.tensor([0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0, 1e4, -1e4], dtype=torch.float64)])
    x = u.float().to(DEV).contiguous()
    y = dmel.dmel_debug_gelu(x).double().cpu()
    xe = x.double().cpu()
    exact = xe * 0.5 * torch.erfc(-xe / math.sqrt(2.0))
    err = (y - exact).abs()
    bound = xe.abs() * (7.5e-8 + 4e-7) + 1.2e-7 * exact.abs() + 1e-37
    worst = float((err / bound).max())
    print(f"gelu: worst error / bound {worst:.3f}, max abs error {float(err.max()):.2e}")
    assert worst <= 1.0
    assert float(y[-2]) == 1e4 and float(y[-1]) == 0.0  # saturated tails are exact


@pytest.mark.parametrize("m,k,n,lda", [
    (1, 8, 8, 8),             # one row, one K step (zero-filled past K), one column group
    (300, 136, 200, 136),     # ragged in every dimension: a half-empty second CTA pair, a partial column tile
    (4096, 512, 1536, 512),   # 192-column tiles, 16 x 8 = 128 of them: more than one per cluster on 148 SMs
    (257, 6144, 392, 6200),   # the hMLP's K; A a row slice of a wider array
    (1600, 256, 6144, 256),   # the last stage's shape: 256-column tiles (fewer rounds of tiles)
    (25599, 72, 1528, 72),    # 256-column tiles, ragged rows, columns and K, 9 rounds of tiles
])
def test_stage_gemm_matches_fp64(m, k, n, lda):
    """The tcgen05 stage GEMM alone against an fp64 product of the same bf16 inputs: fp32 sums of
    k products differ from the exact sum by rounding only (bound ~k * 2^-24 of the sum of
    |a_i b_i|)."""
    g = torch.Generator(device=DEV).manual_seed(97)
    a_full = torch.randn((m, lda), device=DEV, generator=g).to(torch.bfloat16)
    a = a_full[:, :k]
    b = torch.randn((k, n), device=DEV, generator=g).to(torch.bfloat16)
    c = torch.full((m, n), float("nan"), device=DEV)
    dmel.dmel_debug_gemm(a, b, c)
    torch.cuda.synchronize()
    assert dmel.dmel_get_device_error(clear=True) == 0
    ad, bd = a.double().cpu(), b.double().cpu()
    ref = ad @ bd
    bound = (ad.abs() @ bd.abs()) * (k * 2.0 ** -24) + 1e-30
    err = (c.double().cpu() - ref).abs()
    assert torch.isfinite(c).all()
    assert (err <= bound).all(), f"worst excess {(err / bound).max().item():.3g}"
