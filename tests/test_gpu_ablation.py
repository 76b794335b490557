"""The toy experiment ("SVDQuant Smoothing, Low-rank and Residual Quantization",
section "Toy experiment") through the GPU path: each variant's output error from
svdq_prepare + svdq_linear against the float64 oracle's error for the same variant.
The GPU split is randomized and its factors are bf16, so errors agree to a few per
cent rather than exactly; the quantisation error they measure is ~25-50 %."""

import numpy as np
import pytest
import torch

from rank_bit_residual_b200.ablation import ablation
from tests.gpu_util import device
from tests.test_oracle_ablation import errors, toy

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seed", [0, 1])
def test_gpu_ablation_matches_oracle(seed):
    x, W, scale, _, _ = toy(seed)
    dev = device()
    res = ablation(torch.from_numpy(x).to(dev), torch.from_numpy(W).to(dev), torch.from_numpy(scale).to(dev),
                   ranks=range(7), fmt="int4")
    naive, smooth, two = errors(seed)
    assert res["naive"] == pytest.approx(naive, rel=0.05)
    assert res["smooth_only"] == pytest.approx(smooth, rel=0.05)
    for r in range(7):
        assert res["two_branch"][r] == pytest.approx(two[r], rel=0.08), (r, res["two_branch"][r], two[r])
    assert res["two_branch"][0] == res["smooth_only"]
    assert res["two_branch"][6] < res["two_branch"][1] < res["naive"]
    # the singular values it reports are those of W and diag(scale) W
    s_ws = np.linalg.svd(scale[:, None].astype(np.float64) * W, compute_uv=False)
    assert np.allclose(res["sigma_smoothed"], s_ws[:16], rtol=1e-9)
