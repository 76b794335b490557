"""MXFP4: e2m1 elements with one power-of-two (E8M0) scale per 32-element block.
Test infrastructure only (imported by tests/, smoke() and the bench's CPU leg).

The "SVDQuant parameter configuration guide" (msModelSlim), step 2's recommended
configuration, quantises the residual branch and the activations "per_block" as
"mxfp4", "symmetric", method "minmax", without spelling the format out. Reading
(the public OCP microscaling format of that name):

* blocks of 32 consecutive elements along the reduction dim (K = M);
* the block scale is 2^X with X = floor(log2(amax_b)) - 2 (2 = the exponent of
  e2m1's largest value, 6 = 1.5 * 2^2), clamped to [-127, 127], stored as the
  E8M0 byte X + 127; an all-zero block takes X = -127 (byte 0);
* elements are e2m1 (see oracle.nvfp4) of z / 2^X, round-to-nearest-even,
  saturating at +-6: a block whose amax lies in [6 * 2^X, 8 * 2^X) clips its
  largest elements to 6 * 2^X;
* the value is decoded as code * 2^X; there is no global scale (the GEMM's
  scale is 1);
* storage as NVFP4: element 2j in the low nibble of byte j; the scales in the
  128x4 layout of oracle.nvfp4 over [rows, K/32].

The elements are a / div, with div the per-column smoothing scale for the
activation (X_hat = x / scale) and 1 for the residual. The block maximum is
rounded once to fp32, amax_b = fl32(max |a / div|) (the largest IEEE quotient),
and X is taken of it; every code is the exact round-to-nearest-even of
a 2^-X / div onto the e2m1 grid (|a| 2^-X and mid * div are exact doubles).
"""

from __future__ import annotations

import numpy as np

from . import nvfp4 as _nv

BLOCK = 32
E2M1_EMAX = 2


def e8m0_decode(code) -> np.ndarray:
    """2^(code - 127); code 255 is NaN."""
    c = np.asarray(code, dtype=np.int64) & 0xFF
    v = np.ldexp(1.0, (c - 127).astype(np.int64))
    return np.where(c == 255, np.nan, v)


def block_exponent(amax) -> np.ndarray:
    """X = floor(log2(amax)) - 2, clamped to [-127, 127]; -127 for a zero block."""
    a = np.asarray(amax, dtype=np.float64)
    m, e = np.frexp(np.where(a > 0, a, 1.0))      # a = m 2^e, m in [0.5, 1): floor(log2 a) = e - 1
    x = (e.astype(np.int64) - 1) - E2M1_EMAX
    x = np.clip(x, -127, 127)
    return np.where(a > 0, x, -127)


def quantize(a, div=None):
    """MXFP4 codes of the elements a[rows, K] / div[K] (div None: 1), K a multiple of
    32: (codes uint8 [rows, K] one nibble per element, scales uint8 [rows, K/32]
    E8M0 bytes)."""
    a32 = np.asarray(a, dtype=np.float32)
    rows, K = a32.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    amax_b = _nv._block_amax_fp32(a32, div, BLOCK)
    X = block_exponent(amax_b)
    p = np.abs(a32.astype(np.float64)).reshape(rows, K // BLOCK, BLOCK) * \
        np.ldexp(1.0, -X)[:, :, None]                              # exact
    c = 1.0 if div is None else np.asarray(div, dtype=np.float32).astype(np.float64).reshape(
        1, K // BLOCK, BLOCK)
    codes = _nv.e2m1_encode_ratio(p, c, a32.reshape(rows, K // BLOCK, BLOCK) < 0)
    return codes.reshape(rows, K), (X + 127).astype(np.uint8)


def dequantize(codes, sf) -> np.ndarray:
    """float64 values code * 2^X of a [rows, K] code matrix."""
    rows, K = codes.shape
    v = _nv.e2m1_decode(codes).reshape(rows, K // BLOCK, BLOCK) * e8m0_decode(sf)[:, :, None]
    return v.reshape(rows, K)


def product(a_codes, a_sf, w_codes_nk, w_sf) -> np.ndarray:
    """sum_k deq(a)[b, k] deq(w)[n, k], exact in float64 (every block product is a
    small integer times a power of two)."""
    return dequantize(a_codes, a_sf) @ dequantize(w_codes_nk, w_sf).T
