"""Pins for the fp32 code mode and the NVFP4 format oracle."""

import numpy as np
import pytest
import torch

from oracle import codes, nvfp4, prepared
from oracle import svdquant as sq
from synth import make_case, to_bf16


# ----------------------------------------------------------- fp32 code mode
def test_fp32_codes_agree_with_exact_mode_except_flagged():
    wl = make_case(64, 256, 32, rank=4, seed=3)
    q32, s32, near = codes.act_codes_int_fp32(wl.x, wl.scale, 4)
    xs64 = wl.x.astype(np.float64) / wl.scale.astype(np.float64)[None, :]
    q64, s64 = sq.int_quantize(xs64, 4)
    assert abs(float(s32) - s64) <= 2e-7 * s64
    diff = q32.astype(np.int64) != q64
    assert np.all(near[diff])                 # every disagreement is a flagged tie
    assert near.mean() <= 1e-3


def test_fp32_codes_hand_ties():
    # scale = 1, max |x| = 7 at bits = 4 -> s = 1: exact halves tie to even
    x = np.array([[0.5, 1.5, 2.5, -3.5, 7.0, 6.5]], dtype=np.float32)
    q, s, near = codes.act_codes_int_fp32(x, np.ones(6, np.float32), 4)
    assert s == 1.0
    assert q.tolist() == [[0, 2, 2, -4, 7, 6]]
    assert near.tolist() == [[True, True, True, True, False, True]]


def test_fp32_codes_all_zero():
    q, s, near = codes.int_codes_fp32(np.zeros((3, 5), np.float32), 4)
    assert s == 0 and not q.any() and not near.any()


def test_residual_codes_are_k_major():
    rng = np.random.default_rng(0)
    R = rng.standard_normal((8, 3)).astype(np.float32)
    q, s, _ = codes.residual_codes_int_fp32(R, 8)
    assert q.shape == (3, 8)
    q2, s2, _ = codes.int_codes_fp32(R, 8)
    assert s == s2 and np.array_equal(q, q2.T)


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
