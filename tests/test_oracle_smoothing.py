"""The smoothing scale of strength alpha (oracle), pinned by closed forms."""

import numpy as np
import pytest

from oracle.smoothing import smooth_scale


def data(seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((64, 48))
    x[:, 5] *= 30.0
    x[:, 9] = 0.0                      # a dead channel
    W = 0.02 * rng.standard_normal((48, 32))
    W[11] = 0.0                        # a dead weight row
    return x, W


def test_alpha_one_and_zero():
    x, W = data()
    s1 = smooth_scale(x, W, 1.0)       # all of the activation range moves into the weight
    s0 = smooth_scale(x, W, 0.0)       # the weight range moves into the activations
    xmax, wmax = np.abs(x).max(0), np.abs(W).max(1)
    assert np.allclose(s1, np.where(xmax > 0, xmax, 1.0), rtol=1e-15)
    assert np.allclose(s0, np.where(wmax > 0, 1.0 / wmax, 1.0), rtol=1e-15)


def test_half_balances_activation_and_weight_ranges():
    # at alpha = 1/2 the smoothed activation and weight have the same range per channel
    x, W = data(1)
    s = smooth_scale(x, W, 0.5)
    xs = np.abs(x / s[None, :]).max(0)
    ws = np.abs(s[:, None] * W).max(1)
    live = (np.abs(x).max(0) > 0) & (np.abs(W).max(1) > 0)
    assert np.allclose(xs[live], ws[live], rtol=1e-12)
    assert np.allclose(xs[live], np.sqrt(np.abs(x).max(0) * np.abs(W).max(1))[live], rtol=1e-12)


def test_dead_channels_take_one():
    x, W = data()
    s = smooth_scale(x, W, 0.3)
    assert s[9] == pytest.approx(1.0 / np.abs(W[9]).max() ** 0.7)
    assert s[11] == pytest.approx(np.abs(x[:, 11]).max() ** 0.3)


def test_rejects_alpha_out_of_range():
    x, W = data()
    with pytest.raises(ValueError):
        smooth_scale(x, W, 1.5)
