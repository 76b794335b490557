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

Evaluation order. Every stored scalar carries the one fp32 rounding named
below (the activation global scale, a block maximum, the block scale value,
the encode scale); every code is the exact round-to-nearest-even of its real
value onto the e2m1 grid. The elements are a / div, with div the per-column
smoothing scale of the activation (X_hat = x / scale) and 1 for the residual:
  amax_t = fl32(max|a / div|);  gs = fl32(2688 / amax_t)  (unless given)
  amax_b = fl32(max over the block of |a / div|)
  sfv = fl32(fl32(amax_b / 6) * gs);  sf = ue4m3_rne(sfv)
  enc = fl32(gs / dec(sf));  code = e2m1_rne(a * enc / div)   (0 when sf == 0)
The e2m1 decision compares |a| enc with mid * div for the grid midpoints mid;
both products are exact in float64 (24 + 24 and 3 + 24 significant bits), so
it is exact. ``mode="exact"`` instead keeps every scalar in float64.
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


def e2m1_encode_ratio(p, c, negative) -> np.ndarray:
    """e2m1 nibble of the real value +-p / c (p >= 0, c > 0), round to nearest even,
    saturating at 6, zero stored as +0. Exact when p and mid * c are exact doubles."""
    p = np.asarray(p, dtype=np.float64)
    c = np.broadcast_to(np.asarray(c, dtype=np.float64), p.shape)
    mids = 0.5 * (_E2M1_GRID[:-1] + _E2M1_GRID[1:])          # .25 .75 1.25 1.75 2.5 3.5 5
    idx = np.zeros(p.shape, dtype=np.int64)
    for i, mid in enumerate(mids):
        q = mid * c
        # above the midpoint between grid points i and i + 1, or on it when i + 1 is even
        up = (p > q) | ((p == q) & ((i + 1) % 2 == 0))
        idx = np.where(up, i + 1, idx)
    sign = (np.asarray(negative) & (idx != 0)).astype(np.uint8) << 3
    return (sign | idx.astype(np.uint8)).astype(np.uint8)


def _block_amax_fp32(a32: np.ndarray, div, block: int) -> np.ndarray:
    """fl32 of the block maxima of |a / div| (max of the IEEE fp32 quotients)."""
    rows, K = a32.shape
    q = np.abs(a32) if div is None else np.abs(a32) / np.asarray(div, dtype=np.float32)[None, :]
    return np.max(q.astype(np.float32).reshape(rows, K // block, block), axis=2)


def quantize(a, gs=None, mode: str = "fp32", div=None):
    """NVFP4 codes of the elements a[rows, K] / div[K] (div None: 1) with
    16-element blocks along K.

    Returns (codes uint8 [rows, K] one nibble per element, sf uint8 [rows, K/16]
    ue4m3 bytes, gs). K must be a multiple of 16.
    """
    rows, K = np.shape(a)
    if K % BLOCK:
        raise ValueError("K must be a multiple of 16")
    if mode != "fp32":
        z = np.asarray(a, dtype=np.float64)
        if div is not None:
            z = z / np.asarray(div, dtype=np.float64)[None, :]
        if gs is None:
            gs = global_scale(np.max(np.abs(z)) if z.size else 0.0, "exact")
        zb = z.reshape(rows, K // BLOCK, BLOCK)
        sf = ue4m3_encode(np.max(np.abs(zb), axis=2) / 6.0 * gs)
        d = e4m3_decode(sf)
        enc = np.where(d > 0, gs / np.where(d > 0, d, 1.0), 0.0)
        return e2m1_encode(zb * enc[:, :, None]).reshape(rows, K), sf, gs
    a32 = np.asarray(a, dtype=np.float32)
    amax_b = _block_amax_fp32(a32, div, BLOCK)
    if gs is None:
        gs = global_scale(np.max(amax_b) if amax_b.size else 0.0, "fp32")
    gs = np.float32(gs)
    sfv = ((amax_b / np.float32(6.0)).astype(np.float32) * gs).astype(np.float32)
    sf = ue4m3_encode(sfv.astype(np.float64))
    d = e4m3_decode(sf).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        enc = np.where(d > 0, (gs / np.where(d > 0, d, np.float32(1.0))).astype(np.float32),
                       np.float32(0.0)).astype(np.float32)
    p = np.abs(a32.astype(np.float64)).reshape(rows, K // BLOCK, BLOCK) * \
        enc.astype(np.float64)[:, :, None]
    c = 1.0 if div is None else np.asarray(div, dtype=np.float32).astype(np.float64).reshape(
        1, K // BLOCK, BLOCK)
    codes = e2m1_encode_ratio(p, c, a32.reshape(rows, K // BLOCK, BLOCK) < 0)
    return codes.reshape(rows, K), sf, gs


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
