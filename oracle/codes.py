"""Integer codes in fp32 arithmetic, the op order the GPU codes are compared in.

The page-1 grid ("Formula and conventions", item 3) is
s = max|z| / qmax, q = clamp(round_half_even(z / s), -qmax, qmax), with
X_hat = x / scale (item 1). Exact mode (oracle.svdquant) evaluates this in
float64; a GPU evaluates it in fp32. For bit-exact code comparison the oracle
repeats the fp32 evaluation, each step one IEEE fp32 operation:

  xs = fl32(x / scale)          IEEE division, x already fp32 (bf16 upcast is exact)
  m  = max |xs|                 exact in any order
  s  = fl32(m / qmax)
  q  = rint_even(fl32(xs / s)), clamped to [-qmax, qmax]

Elements whose exact quotient lies within one fp32 ulp of a rounding
boundary (k + 1/2) are flagged: a different but still correctly rounded fp32
evaluation could decide them either way, and the comparison reports them.
"""

from __future__ import annotations

import numpy as np

from .svdquant import qmax_of


def _near_half(xs32: np.ndarray, s32: np.float32) -> np.ndarray:
    t = xs32.astype(np.float64) / np.float64(s32)
    frac = t - np.floor(t)
    ulp = np.spacing(np.abs(t).astype(np.float32)).astype(np.float64)
    return np.abs(frac - 0.5) <= ulp


def smooth_fp32(x, scale) -> np.ndarray:
    """X_hat = fl32(x / scale) with IEEE fp32 division, per input channel."""
    x32 = np.asarray(x, dtype=np.float32)
    s32 = np.asarray(scale, dtype=np.float32)
    return (x32 / s32[None, :]).astype(np.float32)


def int_codes_fp32(z32: np.ndarray, bits: int):
    """Per-tensor symmetric INT codes of an fp32 tensor: (codes int8, s fp32, near_tie).

    An all-zero tensor has s = 0 and zero codes.
    """
    z32 = np.asarray(z32, dtype=np.float32)
    qm = np.float32(qmax_of(bits))
    m = np.float32(np.max(np.abs(z32))) if z32.size else np.float32(0.0)
    s = np.float32(m / qm)
    if s == 0:
        return (np.zeros(z32.shape, dtype=np.int8), np.float32(0.0),
                np.zeros(z32.shape, dtype=bool))
    t = (z32 / s).astype(np.float32)
    q = np.clip(np.rint(t), -qm, qm).astype(np.int8)
    return q, s, _near_half(z32, s)


def act_codes_int_fp32(x, scale, bits: int):
    """Activation branch: INT codes of X_hat = x / scale (per tensor)."""
    return int_codes_fp32(smooth_fp32(x, scale), bits)


def residual_codes_int_fp32(R32, bits: int):
    """Residual branch: INT codes of R[M,N], returned K-major as codes[N,M]."""
    q, s, near = int_codes_fp32(np.asarray(R32, dtype=np.float32), bits)
    return np.ascontiguousarray(q.T), s, np.ascontiguousarray(near.T)
