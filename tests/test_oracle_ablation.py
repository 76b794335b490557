"""The toy experiment of "SVDQuant Smoothing, Low-rank and Residual Quantization"
(section "Toy experiment"): one 30x activation channel, naive W4A4 against smoothing
only against the two-branch approximation at ranks 0 to 6, on the float64 oracle.
The page gives no numbers, only the comparison; what it fixes is checked: rank 0 of
the two-branch form is smoothing only, the rank-r branch keeps the weight's leading
directions out of the quantiser so the error drops once it is on, and smoothing moves
the activation outlier into the weight, whose leading singular value then grows."""

import numpy as np

from oracle import svdquant as osv
from synth.workloads import generate


def toy(seed=0):
    return generate(64, 256, 128, seed=seed, x_dist="normal", dtype="fp32", outlier_idx=[37],
                    outlier_factor=30.0, w_std=0.02, spikes=(1.0, 0.8, 0.6, 0.4, 0.3, 0.2), alpha=0.5)


def errors(seed=0):
    x, W, scale, _, _ = toy(seed)
    ref = x.astype(np.float64) @ W.astype(np.float64)
    e = lambda y: float(np.linalg.norm(y - ref) / np.linalg.norm(ref))
    naive = e(osv.svdquant_linear(x, W, np.ones_like(scale), 0, 4))
    smooth = e(osv.svdquant_linear(x, W, scale, 0, 4))
    two = [e(osv.svdquant_linear(x, W, scale, r, 4)) for r in range(7)]
    return naive, smooth, two


def test_rank_zero_two_branch_is_smoothing_only():
    _, smooth, two = errors(0)
    assert two[0] == smooth


def test_low_rank_branch_lowers_the_error():
    for seed in (0, 1, 2):
        naive, smooth, two = errors(seed)
        assert two[1] < 0.8 * smooth, (seed, smooth, two)
        assert two[6] < two[1] < naive, (seed, naive, two)


def test_smoothing_moves_the_outlier_into_the_weight():
    x, W, scale, _, _ = toy(0)
    s_w = np.linalg.svd(W.astype(np.float64), compute_uv=False)
    s_ws = np.linalg.svd(scale[:, None].astype(np.float64) * W, compute_uv=False)
    # relative to the bulk, the leading direction of the smoothed weight stands out more
    assert s_ws[0] / np.median(s_ws) > 1.2 * s_w[0] / np.median(s_w)
