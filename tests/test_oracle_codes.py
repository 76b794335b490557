"""Pins for the INT code mode (exactly rounded quotients, fp32 scales) and the NVFP4
format oracle."""

import numpy as np
import pytest
import torch

from oracle import codes, nvfp4, prepared
from oracle import svdquant as sq
from synth import make_case, to_bf16


# ------------------------------------------------------------- INT code mode
def _definition_codes(x, scale, s, bits):
    """Page-1 grid in float64 with a given s: clamp(rint(x / scale / s))."""
    qm = 2 ** (bits - 1) - 1
    xs64 = np.asarray(x, np.float64) / np.asarray(scale, np.float64)[None, :]
    return np.clip(np.rint(xs64 / np.float64(s)), -qm, qm).astype(np.int64)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_codes_agree_with_float64_definition(bits):
    # the codes of the page's definition, in float64, given the same s: any
    # disagreement must lie within one fp32 ulp of a half-integer, and there
    # may be at most 1e-5 of them
    wl = make_case(512, 2048, 32, rank=4, seed=3 + bits)
    q, s, near = codes.act_codes_int(wl.x, wl.scale, bits)
    q64 = _definition_codes(wl.x, wl.scale, s, bits)
    diff = q.astype(np.int64) != q64
    assert np.all(near[diff])
    assert diff.sum() <= 1e-5 * diff.size
    assert near.mean() <= 1e-5
    # s is the stored fp32 rounding of max|x / scale| / qmax
    xs64 = wl.x.astype(np.float64) / wl.scale.astype(np.float64)[None, :]
    s64 = np.max(np.abs(xs64)) / (2 ** (bits - 1) - 1)
    assert abs(float(s) - s64) <= 2.0 ** -23 * s64


def test_codes_brute_force_rational():
    # every code of a small case by exact rational arithmetic, one element at a
    # time (no float quotient anywhere)
    from fractions import Fraction
    wl = make_case(6, 64, 16, rank=0, seed=11)
    q, s, _ = codes.act_codes_int(wl.x, wl.scale, 4)
    for b in range(wl.x.shape[0]):
        for k in range(wl.x.shape[1]):
            t = Fraction(float(wl.x[b, k])) / (Fraction(float(wl.scale[k])) * Fraction(float(s)))
            want = max(-7, min(7, round(t)))
            assert q[b, k] == want


def test_codes_hand_ties():
    # scale = 1, max |x| = 7 at bits = 4 -> s = 1: exact halves tie to even
    x = np.array([[0.5, 1.5, 2.5, -3.5, 7.0, 6.5]], dtype=np.float32)
    q, s, near = codes.act_codes_int(x, np.ones(6, np.float32), 4)
    assert s == 1.0
    assert q.tolist() == [[0, 2, 2, -4, 7, 6]]
    assert near.tolist() == [[True, True, True, True, False, True]]
    # scale = 0.5 and 4: the tie is in the smoothed value x / scale
    x = np.array([[0.25, 0.75, 10.0, 14.0, 28.0]], dtype=np.float32)
    sc = np.array([0.5, 0.5, 4.0, 4.0, 4.0], dtype=np.float32)
    q, s, _ = codes.act_codes_int(x, sc, 4)
    assert s == 1.0                              # max |x / scale| = 7
    assert q.tolist() == [[0, 2, 2, 4, 7]]       # 0.5 -> 0, 1.5 -> 2, 2.5 -> 2, 3.5 -> 4


def test_codes_decided_exactly_where_fp32_orders_differ():
    # two elements whose quotient x / (scale s) lies within an fp32 ulp of a
    # half-integer (found by search, checked in exact rationals): the first is
    # -99.4999... (a reciprocal-multiply evaluation gives -100), the second
    # -92.5000... (both the two-division and the reciprocal evaluations give -94)
    x = np.array([[-42.75, -27.75]], np.float32)
    sc = np.array([float.fromhex("0x1.294528p+0"), float.fromhex("0x1.9ab1f8p-1")], np.float32)
    q, s, near = codes.act_codes_int(x, sc, 8, s=np.float32(0.37))
    assert q.tolist() == [[-99, -93]]
    assert near.tolist() == [[True, True]]


def test_exact_codes_differ_from_two_roundings_only_at_ties():
    # the fp32 evaluation fl32(fl32(x / scale) / s) rounds twice; its codes may
    # differ from the exactly rounded quotient, but only next to a half-integer
    wl = make_case(256, 1024, 16, rank=0, seed=5)
    q, s, _ = codes.act_codes_int(wl.x, wl.scale, 8)
    q32, s32 = codes.act_codes_int_ieee32(wl.x, wl.scale, 8)
    assert s32 == s
    t = wl.x.astype(np.float64) / (wl.scale.astype(np.float64)[None, :] * np.float64(s))
    diff = q != q32
    dist = np.abs(t - np.floor(t) - 0.5)
    assert np.all(dist[diff] <= 2.0 * np.spacing(np.abs(t[diff]).astype(np.float32)))


def test_codes_all_zero():
    q, s, near = codes.int_codes(np.zeros((3, 5), np.float32), 4)
    assert s == 0 and not q.any() and not near.any()
    q, s, near = codes.act_codes_int(np.zeros((2, 4), np.float32), np.ones(4, np.float32), 4)
    assert s == 0 and not q.any()


def test_residual_codes_are_k_major():
    rng = np.random.default_rng(0)
    R = rng.standard_normal((8, 3)).astype(np.float32)
    q, s, _ = codes.residual_codes_int(R, 8)
    assert q.shape == (3, 8)
    q2, s2, _ = codes.int_codes(R, 8)
    assert s == s2 and np.array_equal(q, q2.T)
    assert s == np.float32(np.float32(np.max(np.abs(R))) / np.float32(127))


# ---------------------------------------------------------------- formats
def test_e2m1_table(golden):
    g = golden("nvfp4_formats.json")
    vals = nvfp4.e2m1_decode(np.arange(16))
    assert vals.tolist() == g["e2m1_values"]
    assert np.array_equal(np.signbit(vals[8:]), np.ones(8, bool))


def test_e2m1_rounding_ties(golden):
    g = golden("nvfp4_formats.json")["e2m1_round"]
    assert nvfp4.e2m1_encode(np.array(g["inputs"])).tolist() == g["codes"]


def test_e2m1_roundtrip_and_nearest():
    vals = nvfp4.e2m1_decode(np.arange(16))
    enc = nvfp4.e2m1_encode(vals)
    assert np.array_equal(nvfp4.e2m1_decode(enc), vals)     # -0 comes back as +0, value equal
    rng = np.random.default_rng(1)
    v = rng.uniform(-7, 7, 5000)
    dec = nvfp4.e2m1_decode(nvfp4.e2m1_encode(v))
    grid = nvfp4.e2m1_decode(np.arange(16))
    nearest = np.min(np.abs(np.clip(v, -6, 6)[:, None] - grid[None, :]), axis=1)
    assert np.all(np.abs(dec - np.clip(v, -6, 6)) <= nearest + 1e-15)


def test_e4m3_decode_points_and_library(golden):
    g = golden("nvfp4_formats.json")["e4m3_points"]
    assert nvfp4.e4m3_decode(np.array(g["codes"])).tolist() == g["values"]
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = nvfp4.e4m3_decode(np.arange(256))
    assert np.array_equal(np.isnan(lib), np.isnan(ours))
    ok = ~np.isnan(lib)
    assert np.array_equal(lib[ok], ours[ok])


def test_ue4m3_rounding(golden):
    g = golden("nvfp4_formats.json")["ue4m3_round"]
    assert nvfp4.ue4m3_encode(np.array(g["inputs"])).tolist() == g["codes"]
    # in-range values agree with the library's round-to-nearest-even conversion
    rng = np.random.default_rng(2)
    v = np.exp(rng.uniform(np.log(2.0 ** -9), np.log(440.0), 20000)).astype(np.float32)
    lib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(nvfp4.ue4m3_encode(v), lib)


# ------------------------------------------------------- block quantisation
def test_nvfp4_block_quantisation_consistency():
    rng = np.random.default_rng(4)
    z = (rng.standard_t(3, (40, 128)) * 0.3).astype(np.float32)
    c, sf, gs = nvfp4.quantize(z)
    assert c.shape == z.shape and sf.shape == (40, 8) and c.max() <= 15
    amax = np.max(np.abs(z))
    assert gs == np.float32(np.float32(2688.0) / np.float32(amax))
    deq = nvfp4.dequantize(c, sf, gs)
    # each element lies within half of its block's largest grid step (2 * sf / gs),
    # plus the scale's own rounding for the block maximum
    step = 2.0 * nvfp4.e4m3_decode(sf) / float(gs)
    err = np.abs(deq - z).reshape(40, 8, 16)
    amax_b = np.max(np.abs(z).reshape(40, 8, 16), axis=2)
    assert np.all(err <= (0.5 * step + amax_b * 2.0 ** -3)[:, :, None] + 1e-12)
    # the tensor maximum maps to +-6 with block scale at (or 1 ulp below) 448
    i = np.unravel_index(np.argmax(np.abs(z)), z.shape)
    assert nvfp4.e2m1_decode(c[i]) in (6.0, -6.0)


def test_nvfp4_zero_blocks_and_given_global_scale():
    z = np.zeros((2, 32), np.float32); z[1, 16:] = np.linspace(-1, 1, 16)
    c, sf, gs = nvfp4.quantize(z)
    assert sf[0].tolist() == [0, 0] and sf[1, 0] == 0 and not c[0].any() and not c[1, :16].any()
    c2, sf2, gs2 = nvfp4.quantize(z, gs=np.float32(100.0))
    assert gs2 == np.float32(100.0)
    assert nvfp4.quantize(np.zeros((1, 16), np.float32))[2] == 1.0


def test_nvfp4_representable_values_roundtrip():
    # block max 6 and gs with sf exactly 1: every e2m1 value round-trips
    vals = nvfp4.e2m1_decode(np.arange(16)).astype(np.float32)
    z = np.tile(vals, (1, 1))
    c, sf, gs = nvfp4.quantize(z, gs=np.float32(1.0))
    assert nvfp4.e4m3_decode(sf).tolist() == [[1.0]]
    assert np.array_equal(nvfp4.dequantize(c, sf, gs), vals.astype(np.float64)[None, :])


def test_nvfp4_exact_and_fp32_modes_close():
    rng = np.random.default_rng(5)
    z = rng.standard_normal((16, 64)).astype(np.float32)
    c32, sf32, _ = nvfp4.quantize(z, mode="fp32")
    c64, sf64, _ = nvfp4.quantize(z, mode="exact")
    assert (c32 != c64).mean() < 0.01 and (sf32 != sf64).mean() < 0.05


def test_e2m1_ratio_ties_go_to_even():
    # p / c exactly on a midpoint, with divisors whose quotient a float division
    # could not land on exactly: the even neighbour wins
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    even = [0, 2, 2, 4, 4, 6, 6]                  # e2m1 indices: 0 1 | 1 1.5 -> 1 ...
    for c in (1.0, 0.1, 3.0, 1.0 / 3.0, 7.3):
        c32 = float(np.float32(c))
        p = np.array([m * c32 for m in mids])        # exact: mid has <= 3 significant bits
        got = nvfp4.e2m1_encode_ratio(p, c32, np.zeros(7, bool))
        assert got.tolist() == even, c
        neg = nvfp4.e2m1_encode_ratio(p, c32, np.ones(7, bool))
        assert neg.tolist() == [0] + [8 | e for e in even[1:]]
    # just off the midpoint goes to the nearer point; saturation above 6
    up = nvfp4.e2m1_encode_ratio(np.nextafter(np.array([0.25, 5.0]), 10), 1.0, np.zeros(2, bool))
    assert up.tolist() == [1, 7]
    assert nvfp4.e2m1_encode_ratio(np.array([100.0]), 1.0, np.zeros(1, bool)).tolist() == [7]


def _fr(v):
    from fractions import Fraction
    return Fraction(float(v))


def _e2m1_index_exact(t):
    """RNE index of a non-negative Fraction onto {0,.5,1,1.5,2,3,4,6}, saturating."""
    grid = [_fr(g) for g in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
    if t >= grid[-1]:
        return 7
    best = min(range(8), key=lambda i: (abs(t - grid[i]), i % 2))
    return best


@pytest.mark.parametrize("with_div", [False, True])
def test_nvfp4_quantize_brute_force(with_div):
    # block maxima, scales and every code of a small case, element by element in
    # exact rationals (the scalars carry their stated fp32 roundings)
    rng = np.random.default_rng(12)
    a = (rng.standard_normal((3, 48)) * 3).astype(np.float32)
    div = rng.uniform(0.3, 3.0, 48).astype(np.float32) if with_div else None
    c, sf, gs = nvfp4.quantize(a, div=div)
    d = np.ones(48, np.float32) if div is None else div
    q32 = (np.abs(a) / d[None, :]).astype(np.float32)
    assert gs == np.float32(np.float32(2688.0) / np.float32(q32.max()))
    for r in range(3):
        for b in range(3):
            amax = np.float32(q32[r, 16 * b:16 * b + 16].max())
            sfv = np.float32(np.float32(amax / np.float32(6.0)) * gs)
            assert sf[r, b] == nvfp4.ue4m3_encode(np.array([sfv], np.float64))[0]
            dec = np.float32(nvfp4.e4m3_decode(sf[r, b]))
            enc = np.float32(gs / dec) if dec > 0 else np.float32(0.0)
            for k in range(16 * b, 16 * b + 16):
                t = abs(_fr(a[r, k])) * _fr(enc) / _fr(d[k])
                idx = _e2m1_index_exact(t)
                want = idx | (8 if (a[r, k] < 0 and idx) else 0)
                assert c[r, k] == want, (r, k)


@pytest.mark.parametrize("with_div", [False, True])
def test_mxfp4_quantize_brute_force(with_div):
    from oracle import mxfp4
    rng = np.random.default_rng(13)
    a = (rng.standard_normal((3, 64)) * 5).astype(np.float32)
    div = rng.uniform(0.3, 3.0, 64).astype(np.float32) if with_div else None
    c, sf = mxfp4.quantize(a, div=div)
    d = np.ones(64, np.float32) if div is None else div
    q32 = (np.abs(a) / d[None, :]).astype(np.float32)
    import math
    for r in range(3):
        for b in range(2):
            amax = float(q32[r, 32 * b:32 * b + 32].max())
            X = math.floor(math.log2(amax)) - 2
            assert sf[r, b] == X + 127
            for k in range(32 * b, 32 * b + 32):
                t = abs(_fr(a[r, k])) / _fr(d[k]) / _fr(2.0 ** X)
                idx = _e2m1_index_exact(t)
                assert c[r, k] == idx | (8 if (a[r, k] < 0 and idx) else 0), (r, k)


# ------------------------------------------------------------------ layouts
def test_sf_layout_points_and_bijection(golden):
    g = golden("nvfp4_formats.json")["sf_layout"]
    for r, c, off in g["points"]:
        assert nvfp4.sf_offset(r, c, g["rows"], g["kblocks"]) == off
    rows, kb = 200, 11
    rr, cc = np.meshgrid(np.arange(384), np.arange(12), indexing="ij")
    offs = nvfp4.sf_offset(rr, cc, rows, kb).ravel()
    assert np.array_equal(np.sort(offs), np.arange(384 * 12))      # a permutation
    rng = np.random.default_rng(6)
    sf = rng.integers(0, 255, (rows, kb)).astype(np.uint8)
    buf = nvfp4.sf_swizzle(sf)
    assert buf.size == 256 * 12
    assert np.array_equal(nvfp4.sf_unswizzle(buf, rows, kb), sf)


def test_pack_nibbles_order():
    c = np.array([[1, 2, 15, 0]], np.uint8)
    p = nvfp4.pack_nibbles(c)
    assert p.tolist() == [[0x21, 0x0F]]
    assert np.array_equal(nvfp4.unpack_nibbles(p), c)


def test_nvfp4_prepared_product_matches_brute_force():
    rng = np.random.default_rng(7)
    a = (rng.standard_normal((3, 32))).astype(np.float32)
    w = (rng.standard_normal((4, 32))).astype(np.float32)
    ca, sa, ga = nvfp4.quantize(a)
    cw, sw, gw = nvfp4.quantize(w)
    acc = prepared.nvfp4_product(ca, sa, cw, sw)
    for i in range(3):
        for j in range(4):
            s = 0.0
            for k in range(32):
                s += (nvfp4.e2m1_decode(ca[i, k]) * nvfp4.e4m3_decode(sa[i, k // 16]) *
                      nvfp4.e2m1_decode(cw[j, k]) * nvfp4.e4m3_decode(sw[j, k // 16]))
            assert acc[i, j] == s
    # dequantised product approximates the fp32 product
    y = acc / (float(ga) * float(gw))
    assert np.linalg.norm(y - a.astype(np.float64) @ w.T.astype(np.float64)) < 0.25 * np.linalg.norm(a @ w.T)


def test_bf16_rounding_helper_is_rne():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9], np.float32)
    assert to_bf16(v).tolist() == [1.0, 1.0, 1.0 + 2 ** -6, 1.0]
