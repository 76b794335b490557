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


def _mxfp4_errors(seed):
    """The toy experiment with MXFP4 in place of the INT grid (the configuration
    guide's recommended format), on the float64 oracle: smooth, split exactly,
    quantise X_hat and R in 32-element blocks along K."""
    from oracle import mxfp4 as omx
    from oracle import svdquant as osv
    x, W, scale, _, _ = toy(seed)
    ref = x.astype(np.float64) @ W.astype(np.float64)

    def run(s, r):
        xs, ws = osv.smooth_inputs(x, W, s)
        L1, L2, R = osv.split_weight(ws, r)
        ca, sa = omx.quantize(xs)
        cr, sr = omx.quantize(np.ascontiguousarray(R.T))
        y = (xs @ L1) @ L2 + omx.product(ca, sa, cr, sr)
        return float(np.linalg.norm(y - ref) / np.linalg.norm(ref))

    return run(np.ones_like(scale), 0), run(scale, 0), [run(scale, r) for r in range(7)]


def test_gpu_ablation_mxfp4_matches_oracle():
    x, W, scale, _, _ = toy(0)
    dev = device()
    res = ablation(torch.from_numpy(x).to(dev), torch.from_numpy(W).to(dev), torch.from_numpy(scale).to(dev),
                   ranks=range(7), fmt="mxfp4")
    naive, smooth, two = _mxfp4_errors(0)
    assert res["naive"] == pytest.approx(naive, rel=0.05)
    assert res["smooth_only"] == pytest.approx(smooth, rel=0.05)
    for r in range(7):
        assert res["two_branch"][r] == pytest.approx(two[r], rel=0.08), (r, res["two_branch"][r], two[r])
