"""Page-1 contract of the SVDQuant linear, float64 (exact mode).

Source: "SVDQuant Smoothing, Low-rank and Residual Quantization", sections
"Return requirements" and "Formula and conventions". Layout is x[B,M] @ W[M,N]
(not the transposed nn.Linear layout).
"""

from __future__ import annotations

import numbers

import numpy as np


def _f64(a) -> np.ndarray:
    return np.array(a, dtype=np.float64, copy=True)


def check_smoothing(x, weight, scale) -> None:
    """_check_smoothing: nonempty x[B,M], weight[M,N], finite positive scale[M].

    Raises ValueError for any other layout or scale ("Return requirements",
    _check_smoothing).
    """
    x = np.asarray(x)
    w = np.asarray(weight)
    s = np.asarray(scale)
    if x.ndim != 2 or w.ndim != 2:
        raise ValueError("x and weight must be matrices")
    if s.ndim != 1:
        raise ValueError("scale must be a vector")
    if x.size == 0 or w.size == 0 or s.size == 0:
        raise ValueError("empty input")
    if x.shape[1] != w.shape[0]:
        raise ValueError("x[B,M] and weight[M,N] disagree on M")
    if s.shape[0] != w.shape[0]:
        raise ValueError("scale must have M entries")
    s64 = s.astype(np.float64)
    if not np.all(np.isfinite(s64)) or not np.all(s64 > 0):
        raise ValueError("scale must be finite and positive")


def check_rank(weight, rank) -> None:
    """_check_rank: weight is a matrix and rank is a Python int in [0, min(M,N)].

    "Python int" is read as an int that is not a bool ("Return requirements",
    _check_rank).
    """
    w = np.asarray(weight)
    if w.ndim != 2:
        raise ValueError("weight must be a matrix")
    if isinstance(rank, bool) or not isinstance(rank, numbers.Integral) or \
            isinstance(rank, np.generic):
        raise ValueError("rank must be a Python int")
    if rank < 0 or rank > min(w.shape):
        raise ValueError("rank out of range [0, min(M,N)]")


def smooth_inputs(x, weight, scale):
    """Formula item 1: xs = x / scale, ws = scale[:, None] * weight.

    The pair keeps xs @ ws == x @ weight. Inputs are not modified.
    """
    x64, w64, s64 = _f64(x), _f64(weight), _f64(scale)
    return x64 / s64[None, :], s64[:, None] * w64


def split_weight(weight, rank: int):
    """Formula item 2: truncated-SVD split into left[M,r], right[r,N], residual[M,N].

    left @ right is a best rank-r approximation and residual = weight -
    left @ right. The singular values are put on the left factor (the pages
    accept any equivalent factorisation). rank = 0 gives empty factors and the
    whole weight as residual.
    """
    check_rank(weight, rank)
    w = _f64(weight)
    M, N = w.shape
    if rank == 0:
        return np.zeros((M, 0)), np.zeros((0, N)), w.copy()
    U, S, Vt = np.linalg.svd(w, full_matrices=False)
    left = U[:, :rank] * S[None, :rank]
    right = Vt[:rank, :].copy()
    return left, right, w - left @ right


def _check_bits(bits) -> int:
    if isinstance(bits, bool) or not isinstance(bits, numbers.Integral):
        raise ValueError("bits must be an int")
    bits = int(bits)
    if bits < 2 or bits > 8:
        raise ValueError("bits must lie in [2, 8]")
    return bits


def qmax_of(bits: int) -> int:
    """Largest code of the symmetric grid: 2^(bits-1) - 1."""
    return (1 << (_check_bits(bits) - 1)) - 1


def int_quantize(z, bits: int):
    """Per-tensor symmetric INT encoding: (codes, s).

    s = max|z| / qmax and codes = clamp(round_half_even(z / s), -qmax, qmax);
    an all-zero tensor has s = 0 and zero codes (Formula item 3).
    """
    z64 = _f64(z)
    qm = qmax_of(bits)
    if z64.size == 0:
        return np.zeros(z64.shape, dtype=np.int64), 0.0
    s = float(np.max(np.abs(z64))) / qm
    if s == 0.0:
        return np.zeros(z64.shape, dtype=np.int64), 0.0
    q = np.clip(np.rint(z64 / s), -qm, qm).astype(np.int64)
    return q, s


def fake_quantize(z, bits: int) -> np.ndarray:
    """fake_quantize: the dequantised values s * codes (same shape, float64)."""
    q, s = int_quantize(z, bits)
    return s * q.astype(np.float64)


def svdquant_linear(x, weight, scale, rank: int, bits: int = 4) -> np.ndarray:
    """svdquant_linear: Y = (X_hat L1) L2 + Q(X_hat) Q(R).

    Smooth, split the smoothed weight, keep the low-rank branch on the
    unquantised smoothed activations and quantise only the residual branch,
    with one `bits` for both operands (Formula item 3).
    """
    check_smoothing(x, weight, scale)
    check_rank(weight, rank)
    _check_bits(bits)
    xs, ws = smooth_inputs(x, weight, scale)
    L1, L2, R = split_weight(ws, rank)
    return (xs @ L1) @ L2 + fake_quantize(xs, bits) @ fake_quantize(R, bits)


def tail_norm(weight, rank: int) -> float:
    """Frobenius norm of the optimal rank-r residual (Eckart-Young).

    The squared singular values are the eigenvalues of the smaller Gram matrix,
    so the tail is sqrt(sum of all but the r largest of them).
    """
    w = _f64(weight)
    g = w.T @ w if w.shape[0] >= w.shape[1] else w @ w.T
    lam = np.clip(np.sort(np.linalg.eigvalsh(g))[::-1], 0.0, None)
    return float(np.sqrt(np.sum(lam[rank:])))
