"""The two-branch linear evaluated from prepared (stored) operands, float64.

Equation of "Formula and conventions" item 3, Y = (X_hat L1) L2 + Q(X_hat) Q(R),
with the smoothing folded into the down factor the way the NVFP4 operator's
parameters store it ("flashinfer.gemm.svdquant_linear": l2t_smoothed is the
down factor times the per-channel pre-quant scale, shape (k, r)):

  X_hat L1 = (x / scale) (diag(scale) Ld) = x Ld,     Ld = diag(1/scale) L1

so the low-rank branch reads the raw activation. The residual branch is the
dequantised integer (or block-scaled) product of activation and residual codes.

Every quantity is upcast exactly to float64; the integer product is a float64
GEMM of integer codes, exact because every partial sum stays below 2^53.
"""

from __future__ import annotations

import numpy as np

from . import mxfp4, nvfp4


def low_rank(x, ld, lu) -> np.ndarray:
    """(x Ld) Lu with Ld[M, r] and Lu[r, N] in float64."""
    x64 = np.asarray(x, dtype=np.float64)
    return (x64 @ np.asarray(ld, dtype=np.float64)) @ np.asarray(lu, dtype=np.float64)


def int_product(act_codes, w_codes_nk) -> np.ndarray:
    """Exact integer product C_x[B,M] @ C_w[N,M]^T (as float64)."""
    a = np.asarray(act_codes, dtype=np.float64)
    w = np.asarray(w_codes_nk, dtype=np.float64)
    return a @ w.T


def linear_int(x, ld, lu, act_codes, s_x, w_codes_nk, s_w, bias=None) -> np.ndarray:
    """Y = x Ld Lu + s_x s_w (C_x C_w^T) [+ bias]."""
    y = low_rank(x, ld, lu) + (float(s_x) * float(s_w)) * int_product(act_codes, w_codes_nk)
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y


def nvfp4_product(a_codes, a_sf, w_codes_nk, w_sf) -> np.ndarray:
    """Block-scaled product sum_k (a_k sfa) (w_k sfw), codes one nibble per element."""
    B, K = a_codes.shape
    N = w_codes_nk.shape[0]
    A = nvfp4.dequantize(a_codes, a_sf, 1.0)
    W = nvfp4.dequantize(w_codes_nk, w_sf, 1.0)
    assert W.shape == (N, K)
    return A @ W.T


def linear_nvfp4(x, ld, lu, a_codes, a_sf, gs_x, w_codes_nk, w_sf, gs_w, bias=None):
    """Y = x Ld Lu + (1 / (gs_x gs_w)) sum_blocks (a sfa)(w sfw) [+ bias]."""
    y = low_rank(x, ld, lu) + nvfp4_product(a_codes, a_sf, w_codes_nk, w_sf) / (
        float(gs_x) * float(gs_w))
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y


def linear_mxfp4(x, ld, lu, a_codes, a_sf, w_codes_nk, w_sf, bias=None):
    """Y = x Ld Lu + sum_blocks (a 2^Xa)(w 2^Xw) [+ bias]: the MXFP4 variant of
    the same operator (E8M0 block scales per 32 elements, no global scale)."""
    y = low_rank(x, ld, lu) + mxfp4.product(a_codes, a_sf, w_codes_nk, w_sf)
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y
