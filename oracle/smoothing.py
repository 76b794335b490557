"""Smoothing scale of a given migration strength, float64 (test infrastructure only:
imported by tests/, smoke() and the bench's CPU leg, never by the library).

"SVDQuant Smoothing, Low-rank and Residual Quantization" (Formula item 1) takes the
per-channel scale as given; the "SVDQuant parameter configuration guide" (msModelSlim),
step 3 "choose and tune the parameters", tunes its migration strength
(iter_smooth.alpha). Reading: the usual migration scale

    scale_j = max_b |x[b, j]|^alpha / max_n |W[j, n]|^(1 - alpha),

where a factor whose maximum is zero is 1.
"""

from __future__ import annotations

import numpy as np


def smooth_scale(x, W, alpha: float) -> np.ndarray:
    """The scale of strength alpha from calibration activations x [B, M] and W [M, N]."""
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    if not 0.0 <= alpha <= 1.0:
        raise ValueError("alpha must lie in [0, 1]")
    xmax = np.max(np.abs(x), axis=0) if x.shape[0] else np.zeros(W.shape[0])
    wmax = np.max(np.abs(W), axis=1)
    a = np.where(xmax > 0, np.power(np.where(xmax > 0, xmax, 1.0), alpha), 1.0)
    b = np.where(wmax > 0, np.power(np.where(wmax > 0, wmax, 1.0), 1.0 - alpha), 1.0)
    return a / b
