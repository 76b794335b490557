"""Integer codes in fp32 arithmetic, the op order the GPU codes are compared in.

The page-1 grid ("Formula and conventions", item 3) is
s = max|z| / qmax, q = clamp(round_half_even(z / s), -qmax, qmax), with
X_hat = x / scale (item 1). Exact mode (oracle.svdquant) evaluates this in
float64; a GPU evaluates it in fp32, where a division per element costs an
order of magnitude more than a multiply. The fp32 reading used here replaces
the per-element divisions by multiplies with correctly rounded reciprocals,
taken once per column (smoothing) or once per tensor (grid step), and folds
the two per-element factors of the activation into one per-column constant;
every step is one IEEE fp32 operation:

  r_k = fl(1 / scale_k)          once per input channel
  xs  = fl(x * r_k)              X_hat (x already fp32: the bf16 upcast is exact)
  m   = max |xs|                 exact in any order
  s   = fl(m / qmax);  u = fl(1 / s)
  activation codes:  c_k = fl(r_k * u),  q = rint_even(fl(x * c_k))
  residual codes:    q = rint_even(fl(R * u))
  both clamped to [-qmax, qmax]

Each quotient then carries at most four roundings of half an ulp, so it lies
within 4 fp32 ulps of the exact one, and a code can differ from the float64
definition only when the exact quotient lies within 4 ulps of a rounding
boundary (k + 1/2); those elements are flagged, and comparisons report them.
"""

from __future__ import annotations

import numpy as np

from .svdquant import qmax_of


def _near_half(t: np.ndarray) -> np.ndarray:
    """Quotients within 4 fp32 ulps of a half-integer."""
    t = np.asarray(t, dtype=np.float64)
    frac = t - np.floor(t)
    ulp = np.spacing(np.abs(t).astype(np.float32)).astype(np.float64)
    return np.abs(frac - 0.5) <= 4.0 * ulp


def smooth_fp32(x, scale) -> np.ndarray:
    """X_hat = fl(x * fl(1 / scale)) per input channel."""
    x32 = np.asarray(x, dtype=np.float32)
    r32 = (np.float32(1.0) / np.asarray(scale, dtype=np.float32)).astype(np.float32)
    return (x32 * r32[None, :]).astype(np.float32)


def int_codes_fp32(z32: np.ndarray, bits: int, exact_quotient=None):
    """Per-tensor symmetric INT codes of an fp32 tensor: (codes int8, s fp32, near_tie).

    An all-zero tensor has s = 0 and zero codes. `exact_quotient(s)` may supply
    the float64 quotient the near-tie flags are taken on (default z / s).
    """
    z32 = np.asarray(z32, dtype=np.float32)
    qm = np.float32(qmax_of(bits))
    m = np.float32(np.max(np.abs(z32))) if z32.size else np.float32(0.0)
    s = np.float32(m / qm)
    if s == 0:
        return (np.zeros(z32.shape, dtype=np.int8), np.float32(0.0),
                np.zeros(z32.shape, dtype=bool))
    u = np.float32(np.float32(1.0) / s)
    t = (z32 * u).astype(np.float32)
    q = np.clip(np.rint(t), -qm, qm).astype(np.int8)
    tq = exact_quotient(s) if exact_quotient is not None else z32.astype(np.float64) / np.float64(s)
    return q, s, _near_half(tq)


def act_codes_int_fp32(x, scale, bits: int):
    """Activation branch: INT codes of X_hat = x / scale (per tensor).

    The grid step s comes from max|X_hat|; the codes are rint(fl(x * c_k)) with
    c_k = fl(fl(1 / scale_k) * fl(1 / s)). Near-tie flags are taken on the
    exact quotient x / (scale * s).
    """
    x32 = np.asarray(x, dtype=np.float32)
    r32 = (np.float32(1.0) / np.asarray(scale, dtype=np.float32)).astype(np.float32)
    xs = (x32 * r32[None, :]).astype(np.float32)
    qm = np.float32(qmax_of(bits))
    m = np.float32(np.max(np.abs(xs))) if xs.size else np.float32(0.0)
    s = np.float32(m / qm)
    if s == 0:
        return (np.zeros(xs.shape, dtype=np.int8), np.float32(0.0),
                np.zeros(xs.shape, dtype=bool))
    u = np.float32(np.float32(1.0) / s)
    c = (r32 * u).astype(np.float32)
    t = (x32 * c[None, :]).astype(np.float32)
    q = np.clip(np.rint(t), -qm, qm).astype(np.int8)
    exact = np.asarray(x, dtype=np.float64) / (np.asarray(scale, dtype=np.float64)[None, :] * np.float64(s))
    return q, s, _near_half(exact)


def residual_codes_int_fp32(R32, bits: int):
    """Residual branch: INT codes of R[M,N], returned K-major as codes[N,M]."""
    q, s, near = int_codes_fp32(np.asarray(R32, dtype=np.float32), bits)
    return np.ascontiguousarray(q.T), s, np.ascontiguousarray(near.T)
