"""NVFP4 formats and block quantisation, written from the format definitions.

"flashinfer.gemm.svdquant_linear" (Parameters) fixes the storage of the NVFP4
variant: the residual is packed e2m1 (two codes per byte, (n, k/2) uint8),
block scales are ue4m3 bytes in a "128x4 swizzled layout", and the residual
dequantisation and activation global scales are fp32 scalars. The pages do not
spell out the formats or the scale recipe; this module takes the plainest
reading:

* e2m1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; magnitudes
  {0, 0.5, 1, 1.5, 2, 3, 4, 6}; no inf/NaN. Encoding is round-to-nearest-even
  onto that grid, saturating at 6; a value that rounds to zero is stored +0.
* ue4m3: the e4m3 byte (bias 7, max 448, code 0x7F = NaN, no inf) used for
  non-negative block scales; encoding is round-to-nearest-even, saturating.
* blocks are 16 consecutive elements along the reduction dim (K = M);
* global encode scale gs = 448*6 / amax(tensor) (1 when the tensor is zero);
  block scale sf = ue4m3(amax_b / 6 * gs); codes e2m1(z * gs / sf); the value
  is decoded as code * sf / gs, and the GEMM scale is 1 / (gs_x * gs_w).
* packing: element 2j in the low nibble of byte j.
* the 128x4 layout tiles the [rows, K/16] scale matrix into 128-row x 4-column
  atoms of 512 bytes stored atom after atom along K, then along rows; inside an
  atom the byte of (row r, column c) sits at (r % 32) * 16 + (r / 32) * 4 + c.

The recipe (gs and sf above) is parity unpinned by the pages: no page prints
an NVFP4 example. It is pinned by the format tables and by consistency checks.

Two evaluation orders are provided: ``exact`` (float64 everywhere) and
``fp32`` (one IEEE fp32 op per step, the order GPU codes are compared in):
  amax_t = max|z|;  gs = fl32(2688 / amax_t)  (unless given)
  sfv = fl32(fl32(amax_b / 6) * gs);  sf = ue4m3_rne(sfv)
  enc = fl32(gs / dec(sf));  code = e2m1_rne(fl32(z * enc))   (0 when sf == 0)
"""

from __future__ import annotations

import numpy as np

E2M1_MAX = 6.0
E4M3_MAX = 448.0
GS_NUMERATOR = 448.0 * 6.0   # 2688
BLOCK = 16


# ----------------------------------------------------------------- decode tables
def e2m1_decode(code) -> np.ndarray:
    """Value of an e2m1 nibble from its sign / exponent / mantissa fields."""
    c = np.asarray(code, dtype=np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, (e - 1).astype(np.int64)))
    return sign * mag


def e4m3_decode(code) -> np.ndarray:
    """Value of an e4m3 byte (bias 7; exponent 15 with mantissa 7 is NaN)."""
    c = np.asarray(code, dtype=np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6),
                   np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64)))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


_E2M1_GRID = e2m1_decode(np.arange(8))            # 0, .5, 1, 1.5, 2, 3, 4, 6
_E4M3_GRID = e4m3_decode(np.arange(127))          # finite non-negative, increasing


def _rne_onto(a: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the nearest grid point to a >= 0; ties go to the even index; saturating."""
    a = np.asarray(a, dtype=np.float64)
    lo = np.clip(np.searchsorted(grid, a, side="right") - 1, 0, len(grid) - 1)
    hi = np.minimum(lo + 1, len(grid) - 1)
    mid = 0.5 * (grid[lo] + grid[hi])            # exact: grid points are dyadic
    pick_hi = (a > mid) | ((a == mid) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    return np.where(a >= grid[-1], len(grid) - 1, idx)


def e2m1_encode(v) -> np.ndarray:
    """Round-to-nearest-even e2m1 nibble, saturating at +-6, zero stored as +0."""
    v = np.asarray(v, dtype=np.float64)
    mag = _rne_onto(np.abs(v), _E2M1_GRID).astype(np.uint8)
    sign = ((v < 0) & (mag != 0)).astype(np.uint8) << 3
    return (sign | mag).astype(np.uint8)


def ue4m3_encode(v) -> np.ndarray:
    """Round-to-nearest-even e4m3 byte of a non-negative value, saturating at 448."""
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0) or np.any(np.isnan(v)):
        raise ValueError("ue4m3 scales are non-negative and finite")
    return _rne_onto(v, _E4M3_GRID).astype(np.uint8)


# ------------------------------------------------------------ block quantisation
def global_scale(amax, mode: str = "fp32"):
    """gs = 448*6 / amax (1 for an all-zero tensor)."""
    if mode == "fp32":
        a = np.float32(amax)
        return np.float32(1.0) if a == 0 else np.float32(np.float32(GS_NUMERATOR) / a)
    a = float(amax)
    return 1.0 if a == 0 else GS_NUMERATOR / a


def quantize(z, gs=None, mode: str = "fp32"):
    """NVFP4 codes of z[rows, K] with 16-element blocks along K.

    Returns (codes uint8 [rows, K] one nibble per element, sf uint8 [rows, K/16]
    ue4m3 bytes, gs). K must be a multiple of 16.
    """
    if mode == "fp32":
        z = np.asarray(z, dtype=np.float32)
        ft = np.float32
    else:
        z = np.asarray(z, dtype=np.float64)
        ft = np.float64
    rows, K = z.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 16")
    if gs is None:
        gs = global_scale(np.max(np.abs(z)) if z.size else 0.0, mode)
    gs = ft(gs)
    zb = z.reshape(rows, K // BLOCK, BLOCK)
    amax_b = np.max(np.abs(zb), axis=2)
    sfv = ((amax_b / ft(6.0)).astype(ft) * gs).astype(ft)
    sf = ue4m3_encode(sfv.astype(np.float64))
    d = e4m3_decode(sf).astype(ft)
    with np.errstate(divide="ignore", invalid="ignore"):
        enc = np.where(d > 0, (gs / np.where(d > 0, d, ft(1.0))).astype(ft), ft(0.0)).astype(ft)
    scaled = (zb * enc[:, :, None]).astype(ft)
    codes = e2m1_encode(scaled.astype(np.float64)).reshape(rows, K)
    return codes, sf, gs


def dequantize(codes, sf, gs) -> np.ndarray:
    """float64 values code * sf / gs of a [rows, K] code matrix."""
    rows, K = codes.shape
    v = e2m1_decode(codes).reshape(rows, K // BLOCK, BLOCK) * e4m3_decode(sf)[:, :, None]
    return v.reshape(rows, K) / float(gs)


# ------------------------------------------------------------ storage layouts
def pack_nibbles(codes) -> np.ndarray:
    """[rows, K] nibbles -> [rows, K/2] bytes, element 2j in the low nibble of byte j."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)


def unpack_nibbles(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def sf_padded_shape(rows: int, kblocks: int):
    """Rows padded to 128 and scale columns padded to 4 (the atom shape)."""
    return ((rows + 127) // 128) * 128, ((kblocks + 3) // 4) * 4


def sf_offset(r, c, rows: int, kblocks: int):
    """Byte offset of scale (row r, column c) in the 128x4 swizzled layout."""
    _, kbp = sf_padded_shape(rows, kblocks)
    r = np.asarray(r, dtype=np.int64)
    c = np.asarray(c, dtype=np.int64)
    atom = (r // 128) * (kbp // 4) + (c // 4)
    return atom * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4)


def sf_swizzle(sf) -> np.ndarray:
    """Row-major [rows, K/16] scales -> flat swizzled buffer (padding stays zero)."""
    sf = np.asarray(sf, dtype=np.uint8)
    rows, kb = sf.shape
    rp, kbp = sf_padded_shape(rows, kb)
    out = np.zeros(rp * kbp, dtype=np.uint8)
    r, c = np.meshgrid(np.arange(rows), np.arange(kb), indexing="ij")
    out[sf_offset(r, c, rows, kb)] = sf
    return out


def sf_unswizzle(buf, rows: int, kblocks: int) -> np.ndarray:
    """Flat swizzled buffer -> row-major [rows, K/16] scales."""
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    r, c = np.meshgrid(np.arange(rows), np.arange(kblocks), indexing="ij")
    return buf[sf_offset(r, c, rows, kblocks)]
