"""Activation pass on the GPU against the oracle: INT and NVFP4 codes bit-exact (up to
flagged near-ties), the per-tensor scale bit-exact, and the fused down-projection."""

import numpy as np
import pytest
import torch

import rank_bit_residual_b200 as rb
from oracle import codes as ocodes
from oracle import mxfp4 as omx
from oracle import nvfp4 as onv
from synth import make_case, to_bf16
from tests.gpu_util import assert_codes_match, device, to_dev, x_tensor, rel_fro

pytestmark = pytest.mark.gpu

SHAPES = [(1, 32), (17, 96), (128, 256), (300, 1024), (129, 3072)]


@pytest.mark.parametrize("B,M", SHAPES)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("bits", [4, 8, 2])
def test_int_codes_and_scale(B, M, dtype, bits):
    wl = make_case(B, M, 16, rank=0, seed=B + M + bits, dtype=dtype)
    codes, sf, s, down = rb.svdq_quantize_act(x_tensor(wl), to_dev(wl.scale, torch.float32), f"int{bits}")
    q, s_o, near = ocodes.act_codes_int(wl.x, wl.scale, bits)
    assert np.float32(s.item()) == s_o, (s.item(), s_o)
    assert_codes_match(codes.cpu().numpy(), q, near, f"B={B} M={M} {dtype} int{bits}")
    assert sf is None and down is None


@pytest.mark.parametrize("B,M", SHAPES)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("given_gs", [False, True])
def test_nvfp4_codes_scales_and_layout(B, M, dtype, given_gs):
    wl = make_case(B, M, 16, rank=0, seed=7 * B + M, dtype=dtype)
    gs = np.float32(1234.5) if given_gs else None
    gs_t = to_dev(np.array([gs], np.float32), torch.float32) if given_gs else None
    codes, sf, g, _ = rb.svdq_quantize_act(x_tensor(wl), to_dev(wl.scale, torch.float32), "nvfp4",
                                           act_global_scale=gs_t)
    c_o, sf_o, g_o = onv.quantize(wl.x, gs=gs, div=wl.scale)
    assert np.float32(g.item()) == np.float32(g_o)
    got_sf = sf.cpu().numpy()
    want_sf = onv.sf_swizzle(sf_o)
    assert got_sf.shape == want_sf.shape
    assert np.array_equal(got_sf, want_sf), f"{int((got_sf != want_sf).sum())} scale bytes differ"
    got = onv.unpack_nibbles(codes.cpu().numpy())
    assert np.array_equal(got, c_o), f"{int((got != c_o).sum())} nibbles differ"


@pytest.mark.parametrize("B,M,rank", [(1, 64, 1), (17, 96, 16), (200, 512, 40), (129, 3072, 32),
                                      (64, 256, 256)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_down_projection(B, M, rank, dtype):
    wl = make_case(B, M, 16, rank=0, seed=3 * B + rank, dtype=dtype)
    rp = (rank + 15) // 16 * 16
    rng = np.random.default_rng(rank)
    ld = np.zeros((rp, M), np.float32)
    ld[:rank] = to_bf16(rng.standard_normal((rank, M)).astype(np.float32) * 0.1)
    ld_t = to_dev(ld, torch.bfloat16 if dtype == "bf16" else torch.float32)
    codes, _, s, down = rb.svdq_quantize_act(x_tensor(wl), to_dev(wl.scale, torch.float32), "int4", ld=ld_t)
    d = down.float().cpu().numpy().astype(np.float64)
    got = d[:, :rp] + d[:, rp:]
    want = wl.x.astype(np.float64) @ ld.T.astype(np.float64)
    # bf16 x: exact products, fp32 sums; fp32 x: tf32 operands (10-bit mantissa)
    tol = 2e-5 if dtype == "bf16" else 3e-3
    assert rel_fro(got, want) <= tol, rel_fro(got, want)
    q, s_o, near = ocodes.act_codes_int(wl.x, wl.scale, 4)
    assert np.float32(s.item()) == s_o
    assert_codes_match(codes.cpu().numpy(), q, near)


def test_empty_batch_is_a_no_op():
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device=device())
    codes, sf, s, down = rb.svdq_quantize_act(x, torch.ones(64, device=device()), "int4")
    assert codes.shape == (0, 64)


# long batches (B >= 1024) take the row-slab kernels: ragged last slab, M not a
# multiple of the chunk width, both input types
LONG = [(1024, 256), (1100, 96), (2048, 3072)]


@pytest.mark.parametrize("B,M", LONG)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("bits", [4, 8])
def test_long_batch_int_codes_and_scale(B, M, dtype, bits):
    wl = make_case(B, M, 16, rank=0, seed=B + M + bits, dtype=dtype)
    codes, sf, s, down = rb.svdq_quantize_act(x_tensor(wl), to_dev(wl.scale, torch.float32), f"int{bits}")
    q, s_o, near = ocodes.act_codes_int(wl.x, wl.scale, bits)
    assert np.float32(s.item()) == s_o, (s.item(), s_o)
    assert_codes_match(codes.cpu().numpy(), q, near, f"B={B} M={M} {dtype} int{bits}")


def near_tie_case(B, M, bits, dtype, seed):
    """x and scale with thousands of quotients x / (scale s) at or next to a
    half-integer: s = 1 (x[0, 0] = qmax at scale 1 is the maximum), columns 1-16
    hold exact half-integers at scale 1 (ties to even), and every later column has
    one element, its largest, tuned through its scale to within 2^-19 of a
    half-integer (the others of the column stay below it in magnitude)."""
    rng = np.random.default_rng(seed)
    qm = ocodes.qmax_of(bits)
    x = rng.standard_normal((B, M)).astype(np.float32)
    if dtype == "bf16":
        x = to_bf16(x)
    scale = np.ones(M, np.float32)
    x[:, 0] = 0.0
    x[0, 0] = qm
    for k in range(1, 17):
        col = np.clip(np.round(x[:, k] * 2) / 2, -qm + 0.5, qm - 0.5)
        x[:, k] = np.where(col == np.floor(col), col + 0.5, col).astype(np.float32)
    for k in range(17, M):
        r = int(np.argmax(np.abs(x[:, k])))
        t = (rng.integers(0, qm) + 0.5 + rng.choice([0.0, 1.0, -1.0]) * rng.uniform(0, 2.0 ** -19)) * np.sign(x[r, k])
        scale[k] = np.float32(x[r, k] / t)
    return x, scale


@pytest.mark.parametrize("B,M", [(100, 3072), (300, 3072), (1700, 12288)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("bits", [4, 8])
def test_int_codes_exact_at_half_integers(B, M, dtype, bits):
    """Every code equals round_half_even(x / (scale s)) of the exact quotient, also
    where it lies within an fp32 ulp of a half-integer ("SVDQuant Smoothing,
    Low-rank and Residual Quantization", Formula and conventions item 3: ties to
    even): the estimate x c_k must send each such element to the exact decision.
    B = 100 runs the short-batch pass, 300 the K-split units, 1700 x 12288 the
    flat partition."""
    x, scale = near_tie_case(B, M, bits, dtype, seed=B + bits)
    xt = to_dev(x, torch.bfloat16 if dtype == "bf16" else torch.float32)
    codes, sf, s, down = rb.svdq_quantize_act(xt, to_dev(scale, torch.float32), f"int{bits}")
    q, s_o, near = ocodes.act_codes_int(x, scale, bits)
    assert s_o == np.float32(1.0) and np.float32(s.item()) == s_o, (s.item(), s_o)
    assert int(near.sum()) >= 16 * B, int(near.sum())   # the case does reach the ties
    got = codes.cpu().numpy()
    bad = np.argwhere(got != q)
    assert bad.size == 0, f"{len(bad)} codes differ from the exact rounding, e.g. {bad[:4].tolist()}"


@pytest.mark.parametrize("B,M", LONG)
@pytest.mark.parametrize("given_gs", [False, True])
def test_long_batch_nvfp4_codes_scales_and_layout(B, M, given_gs):
    wl = make_case(B, M, 16, rank=0, seed=3 * B + M)
    gs = np.float32(777.25) if given_gs else None
    gs_t = to_dev(np.array([gs], np.float32), torch.float32) if given_gs else None
    codes, sf, g, _ = rb.svdq_quantize_act(x_tensor(wl), to_dev(wl.scale, torch.float32), "nvfp4",
                                           act_global_scale=gs_t)
    c_o, sf_o, g_o = onv.quantize(wl.x, gs=gs, div=wl.scale)
    assert np.float32(g.item()) == np.float32(g_o)
    assert np.array_equal(sf.cpu().numpy(), onv.sf_swizzle(sf_o))
    assert np.array_equal(onv.unpack_nibbles(codes.cpu().numpy()), c_o)


@pytest.mark.parametrize("B,M,rank", [(1024, 512, 32), (1100, 96, 256), (2048, 3072, 40)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_long_batch_down_projection(B, M, rank, dtype):
    wl = make_case(B, M, 16, rank=0, seed=5 * B + rank, dtype=dtype)
    rp = (rank + 15) // 16 * 16
    rng = np.random.default_rng(rank + 1)
    ld = np.zeros((rp, M), np.float32)
    ld[:rank] = to_bf16(rng.standard_normal((rank, M)).astype(np.float32) * 0.1)
    ld_t = to_dev(ld, torch.bfloat16 if dtype == "bf16" else torch.float32)
    codes, _, s, down = rb.svdq_quantize_act(x_tensor(wl), to_dev(wl.scale, torch.float32), "int4", ld=ld_t)
    d = down.float().cpu().numpy().astype(np.float64)
    got = d[:, :rp] + d[:, rp:]
    want = wl.x.astype(np.float64) @ ld.T.astype(np.float64)
    tol = 2e-5 if dtype == "bf16" else 3e-3
    assert rel_fro(got, want) <= tol, rel_fro(got, want)
    q, s_o, near = ocodes.act_codes_int(wl.x, wl.scale, 4)
    assert np.float32(s.item()) == s_o
    assert_codes_match(codes.cpu().numpy(), q, near)


# long units (many stats-kernel sub-chunks per unit, ring refills) and short
# ones, both input types; two calls in a row on the same workspace
@pytest.mark.parametrize("B,M,dtype", [(2048, 16384, "bf16"), (2048, 3072, "f32"), (2048, 3072, "bf16")])
def test_large_batch_units_long_and_short(B, M, dtype):
    wl = make_case(B, M, 16, rank=0, seed=B + M, dtype=dtype)
    rank = 32
    rng = np.random.default_rng(9)
    ld = to_bf16(rng.standard_normal((rank, M)).astype(np.float32) * 0.1)
    ld_t = to_dev(ld, torch.bfloat16 if dtype == "bf16" else torch.float32)
    for _ in range(2):
        codes, _, s, down = rb.svdq_quantize_act(x_tensor(wl), to_dev(wl.scale, torch.float32), "int4", ld=ld_t)
        q, s_o, near = ocodes.act_codes_int(wl.x, wl.scale, 4)
        assert np.float32(s.item()) == s_o
        assert_codes_match(codes.cpu().numpy(), q, near, f"B={B} M={M} {dtype}")
        d = down.float().cpu().numpy().astype(np.float64)
        got = d[:, :rank] + d[:, rank:]
        want = wl.x.astype(np.float64) @ ld.T.astype(np.float64)
        tol = 2e-5 if dtype == "bf16" else 3e-3
        assert rel_fro(got, want) <= tol, rel_fro(got, want)


# MXFP4: codes and E8M0 scales bit-exact (a power-of-two scale leaves no
# rounding but the smoothing's own), act_scale 1, both batch paths
@pytest.mark.parametrize("B,M", SHAPES + LONG)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_mxfp4_codes_scales_and_layout(B, M, dtype):
    wl = make_case(B, M, 16, rank=0, seed=11 * B + M, dtype=dtype)
    codes, sf, g, _ = rb.svdq_quantize_act(x_tensor(wl), to_dev(wl.scale, torch.float32), "mxfp4")
    c_o, sf_o = omx.quantize(wl.x, div=wl.scale)
    assert g.item() == 1.0
    got_sf = sf.cpu().numpy()
    want_sf = onv.sf_swizzle(sf_o)
    assert got_sf.shape == want_sf.shape
    assert np.array_equal(got_sf, want_sf), f"{int((got_sf != want_sf).sum())} scale bytes differ"
    got = onv.unpack_nibbles(codes.cpu().numpy())
    assert np.array_equal(got, c_o), f"{int((got != c_o).sum())} nibbles differ"


@pytest.mark.parametrize("B,M,rank", [(17, 96, 16), (1100, 96, 256), (2048, 3072, 40)])
def test_mxfp4_down_projection_is_unscaled(B, M, rank):
    wl = make_case(B, M, 16, rank=0, seed=B + rank)
    rp = (rank + 15) // 16 * 16
    rng = np.random.default_rng(rank + 2)
    ld = np.zeros((rp, M), np.float32)
    ld[:rank] = to_bf16(rng.standard_normal((rank, M)).astype(np.float32) * 0.1)
    _, _, g, down = rb.svdq_quantize_act(x_tensor(wl), to_dev(wl.scale, torch.float32), "mxfp4",
                                         ld=to_dev(ld, torch.bfloat16))
    d = down.float().cpu().numpy().astype(np.float64)
    want = wl.x.astype(np.float64) @ ld.T.astype(np.float64)
    assert g.item() == 1.0
    assert rel_fro(d[:, :rp] + d[:, rp:], want) <= 2e-5


def _mx_edge_rows():
    """32-element blocks at the MXFP4 encoder's boundaries: zero and negative-zero
    blocks, block maxima exactly at and just below powers of two (the exponent's
    floor and the clip to 6 2^X), e2m1 ties, huge and tiny exponents, a
    subnormal block, mixed signs. Every value is bf16-representable."""
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -2.5, -5.0, 4.0] * 3)[:32]
    blocks = [
        np.zeros(32),
        -np.zeros(32),
        np.r_[4.0, np.linspace(-3.0, 3.0, 31)],
        np.r_[8.0, -np.linspace(0.0, 7.0, 31)],
        np.r_[7.96875, np.linspace(-7.0, 7.0, 31)],           # amax just below 8: X = 0, clips to 6
        ties,
        np.r_[2.0 ** 120, np.full(31, 2.0 ** 117)],
        np.r_[-(2.0 ** -120), np.full(31, 2.0 ** -124)],
        np.full(32, 1.0e-39),                                  # subnormal block
        np.r_[6.0, -6.0, np.full(30, 0.125)],
    ]
    row = np.concatenate(blocks)
    return to_bf16(np.stack([row, -row, row[::-1].copy(), np.roll(row, 32)]).astype(np.float32))


@pytest.mark.parametrize("B", [4, 256])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_mxfp4_encoder_edges(B, dtype):
    x = np.tile(_mx_edge_rows(), (B // 4, 1))
    M = x.shape[1]
    ones = np.ones(M, np.float32)
    xt = to_dev(x, torch.float32 if dtype == "f32" else torch.bfloat16)
    codes, sf, g, _ = rb.svdq_quantize_act(xt, to_dev(ones, torch.float32), "mxfp4")
    c_o, sf_o = omx.quantize(x, div=ones)
    assert g.item() == 1.0
    assert np.array_equal(sf.cpu().numpy(), onv.sf_swizzle(sf_o))
    assert np.array_equal(onv.unpack_nibbles(codes.cpu().numpy()), c_o)


def test_mxfp4_residual_encoder_edges():
    R = np.ascontiguousarray(_mx_edge_rows().T)          # [M, 4]: the blocks run along M
    R = np.ascontiguousarray(np.tile(R, (1, 4)))           # N = 16
    codes, sf, g = rb.svdq_quantize_residual(to_dev(R, torch.float32), "mxfp4")
    c_o, sf_o = omx.quantize(np.ascontiguousarray(R.T))
    assert g.item() == 1.0
    assert np.array_equal(sf.cpu().numpy(), onv.sf_swizzle(sf_o))
    assert np.array_equal(onv.unpack_nibbles(codes.cpu().numpy()), c_o)


def _nv_edge_rows():
    """16-element blocks at the NVFP4 encoder's boundaries for a given gs = 1:
    zero and negative-zero blocks, e2m1 ties after the ue4m3 scale, block
    maxima whose scale amax / 6 lands on, between and below ue4m3 values (the
    smallest subnormal 2^-9 and under it), the ue4m3 maximum 448 (amax 2688),
    mixed signs."""
    blocks = [
        np.zeros(16),
        -np.zeros(16),
        np.r_[6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -2.5, -3.5, -5.0, 4.0, -6.0],
        np.r_[2688.0, np.linspace(-2000.0, 2000.0, 15)],
        np.r_[6.0 * 2.0 ** -9, np.full(15, 2.0 ** -10)],
        np.r_[3.0 * 2.0 ** -9, np.full(15, 2.0 ** -11)],      # amax / 6 below the smallest scale
        np.r_[6.5, np.linspace(-6.0, 6.0, 15)],                # amax / 6 between two ue4m3 values
        np.r_[-100.0, np.full(15, 33.0)],
    ]
    row = np.concatenate(blocks)
    return to_bf16(np.stack([row, -row, row[::-1].copy(), np.roll(row, 16)]).astype(np.float32))


@pytest.mark.parametrize("B", [4, 256])
def test_nvfp4_encoder_edges_with_given_global_scale(B):
    x = np.tile(_nv_edge_rows(), (B // 4, 1))
    M = x.shape[1]
    ones = np.ones(M, np.float32)
    gs = to_dev(np.array([1.0], np.float32), torch.float32)
    codes, sf, g, _ = rb.svdq_quantize_act(to_dev(x, torch.float32), to_dev(ones, torch.float32), "nvfp4",
                                           act_global_scale=gs)
    c_o, sf_o, g_o = onv.quantize(x, gs=np.float32(1.0), div=ones)
    assert np.float32(g.item()) == np.float32(g_o)
    assert np.array_equal(sf.cpu().numpy(), onv.sf_swizzle(sf_o))
    assert np.array_equal(onv.unpack_nibbles(codes.cpu().numpy()), c_o)
