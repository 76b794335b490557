"""svdq_smooth_scale on the GPU against the oracle's scale of the same strength, and
the strength selection of the ablation tool."""

import numpy as np
import pytest
import torch

import rank_bit_residual_b200 as rb
from oracle.smoothing import smooth_scale
from rank_bit_residual_b200.ablation import select_alpha
from synth import to_bf16
from tests.gpu_util import device
from tests.test_oracle_ablation import toy

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,M,N", [(1, 32, 16), (300, 1024, 272), (4096, 3072, 128), (0, 64, 32)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("alpha", [0.0, 0.25, 0.5, 1.0])
def test_scale_matches_oracle(B, M, N, dtype, alpha):
    rng = np.random.default_rng(B + M + N)
    x = rng.standard_normal((B, M)).astype(np.float32)
    if B:
        x[:, 3] *= 30.0
        x[:, 7 % M] = 0.0
    W = (0.02 * rng.standard_normal((M, N))).astype(np.float32)
    W[5 % M] = 0.0
    if dtype == "bf16":
        x, W = to_bf16(x), to_bf16(W)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    got = rb.svdq_smooth_scale(torch.from_numpy(x).to(device()).to(tdt),
                               torch.from_numpy(W).to(device()).to(tdt), alpha).cpu().numpy()
    want = smooth_scale(x, W, alpha)
    assert np.allclose(got, want, rtol=2e-6, atol=0), np.max(np.abs(got / want - 1))


def test_scale_strided_input():
    x = torch.randn(64, 256, device=device())
    W = torch.randn(128, 96, device=device()) * 0.02
    got = rb.svdq_smooth_scale(x[:, 64:192], W, 0.5).cpu().numpy()
    want = smooth_scale(x[:, 64:192].cpu().numpy(), W.cpu().numpy(), 0.5)
    assert np.allclose(got, want, rtol=2e-6)


def test_rejects_bad_alpha():
    x = torch.randn(4, 32, device=device())
    W = torch.randn(32, 16, device=device())
    with pytest.raises(ValueError):
        rb.svdq_smooth_scale(x, W, 1.5)


def test_select_alpha_keeps_the_smallest_error():
    x, W, _, _, _ = toy(0)
    dev = device()
    res = select_alpha(torch.from_numpy(x).to(dev), torch.from_numpy(W).to(dev), rank=4,
                       alphas=(0.25, 0.5, 0.75, 0.9))
    errs = res["errors"]
    assert all(np.isfinite(v) and 0 < v < 1 for v in errs.values())
    assert res["error"] == min(errs.values()) and errs[res["alpha"]] == res["error"]
    assert np.allclose(res["scale"].cpu().numpy(), smooth_scale(x, W, res["alpha"]), rtol=2e-6)
