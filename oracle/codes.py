"""Integer codes of the per-tensor grid, decided exactly. Test infrastructure only.

The page-1 grid ("SVDQuant Smoothing, Low-rank and Residual Quantization",
"Formula and conventions", item 3) is

    s = max|z| / qmax,   q = clamp(round_half_even(z / s), -qmax, qmax),

applied to the smoothed activation z = X_hat = x / scale (item 1) and to the
residual z = R. A kernel has to store s as an fp32 number, so this module fixes
the one rounding the stored scale carries and none other:

  m   = fl32(max |z|)          the exact maximum, rounded once to fp32
                               (for X_hat: the max of the IEEE quotients
                               fl32(|x| / scale), since rounding is monotone)
  s   = fl32(m / qmax)         IEEE fp32 division
  q   = round_half_even(z / s) of the exact real quotient, clamped

The codes are thus the definition itself, given the stored s: no intermediate
quotient is rounded. They are computed in float64 (every input is an fp32 or
bf16 value and scale * s is exact in float64) and, for the few elements whose
float64 quotient lies within 2^-40 (relative) of a half-integer, in exact
rational arithmetic (fractions.Fraction).

`near_tie_1ulp` flags the elements whose exact quotient lies within one fp32
ulp of a half-integer: an evaluation that rounds the quotient in fp32 may decide
those either way, and comparisons with such an evaluation report them.

`act_codes_int_ieee32` is the other fp32 reading, kept for comparison: every
step one IEEE fp32 operation, fl32(fl32(x / scale) / s), then rint.
"""

from __future__ import annotations

from fractions import Fraction

import numpy as np

from .svdquant import qmax_of

_TIE_BAND = 2.0 ** -40


def _exact_rne_quotient(a: np.ndarray, d1: np.ndarray, d2) -> np.ndarray:
    """round_half_even(a / (d1 * d2)) elementwise, exactly (float64 arrays of
    exactly representable values; d1 * d2 > 0)."""
    a = np.asarray(a, dtype=np.float64)
    d = np.asarray(d1, dtype=np.float64) * np.float64(d2)       # exact: <= 48 significant bits
    t = a / d
    q = np.rint(t)
    frac = t - np.floor(t)
    suspect = np.abs(frac - 0.5) <= _TIE_BAND * np.maximum(np.abs(t), 1.0)
    if np.any(suspect):
        d1b = np.broadcast_to(np.asarray(d1, dtype=np.float64), a.shape)
        for idx in zip(*np.nonzero(suspect)):
            exact = Fraction(float(a[idx])) / (Fraction(float(d1b[idx])) * Fraction(float(d2)))
            q[idx] = float(round(exact))                         # Fraction rounds half to even
    return q


def near_tie_1ulp(a, d1, d2) -> np.ndarray:
    """Elements whose quotient a / (d1 d2) lies within one fp32 ulp of a half-integer."""
    t = np.asarray(a, dtype=np.float64) / (np.asarray(d1, dtype=np.float64) * np.float64(d2))
    frac = t - np.floor(t)
    ulp = np.spacing(np.abs(t).astype(np.float32)).astype(np.float64)
    return np.abs(frac - 0.5) <= ulp


def int_scale_fp32(m32, bits: int) -> np.float32:
    """s = fl32(m / qmax) for an fp32 maximum m."""
    return np.float32(np.float32(m32) / np.float32(qmax_of(bits)))


def act_max_fp32(x, scale) -> np.float32:
    """fl32(max |x / scale|): the largest IEEE quotient fl32(|x_bk| / scale_k)."""
    x32 = np.asarray(x, dtype=np.float32)
    if x32.size == 0:
        return np.float32(0.0)
    q = np.abs(x32) / np.asarray(scale, dtype=np.float32)[None, :]
    return np.float32(np.max(q))


def act_codes_int(x, scale, bits: int, s=None):
    """Activation branch: (codes int8 [B, M], s fp32, near_tie_1ulp) of X_hat = x / scale.

    s defaults to fl32(fl32(max|X_hat|) / qmax); pass a given s (e.g. a kernel's)
    to take the codes of that grid. An all-zero x has s = 0 and zero codes.
    """
    x64 = np.asarray(x, dtype=np.float32).astype(np.float64)
    sc = np.asarray(scale, dtype=np.float32).astype(np.float64)
    if s is None:
        s = int_scale_fp32(act_max_fp32(x, scale), bits)
    s = np.float32(s)
    if s == 0 or x64.size == 0:
        return (np.zeros(x64.shape, dtype=np.int8), np.float32(0.0),
                np.zeros(x64.shape, dtype=bool))
    qm = qmax_of(bits)
    q = np.clip(_exact_rne_quotient(x64, sc[None, :], s), -qm, qm).astype(np.int8)
    return q, s, near_tie_1ulp(x64, sc[None, :], s)


def int_codes(z32, bits: int, s=None):
    """Per-tensor codes of an fp32 tensor z: (codes int8, s fp32, near_tie_1ulp)."""
    z = np.asarray(z32, dtype=np.float32)
    if s is None:
        s = int_scale_fp32(np.max(np.abs(z)) if z.size else 0.0, bits)
    s = np.float32(s)
    if s == 0 or z.size == 0:
        return np.zeros(z.shape, dtype=np.int8), np.float32(0.0), np.zeros(z.shape, dtype=bool)
    qm = qmax_of(bits)
    z64 = z.astype(np.float64)
    q = np.clip(_exact_rne_quotient(z64, np.ones(1), s), -qm, qm).astype(np.int8)
    return q, s, near_tie_1ulp(z64, np.ones(1), s)


def residual_codes_int(R32, bits: int):
    """Residual branch: INT codes of R[M,N], returned K-major as codes[N,M]."""
    q, s, near = int_codes(R32, bits)
    return np.ascontiguousarray(q.T), s, np.ascontiguousarray(near.T)


def act_codes_int_ieee32(x, scale, bits: int):
    """The two-division fp32 evaluation: q = rint(fl32(fl32(x / scale) / s)), with the
    same s. Differs from act_codes_int only where the quotient is within about two
    fp32 ulps of a half-integer."""
    x32 = np.asarray(x, dtype=np.float32)
    xs = (x32 / np.asarray(scale, dtype=np.float32)[None, :]).astype(np.float32)
    s = int_scale_fp32(np.max(np.abs(xs)) if xs.size else 0.0, bits)
    if s == 0:
        return np.zeros(xs.shape, dtype=np.int8), np.float32(0.0)
    qm = np.float32(qmax_of(bits))
    return np.clip(np.rint((xs / s).astype(np.float32)), -qm, qm).astype(np.int8), s
