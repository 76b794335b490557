"""Residual GEMM + low-rank epilogue on the GPU against the oracle."""

import numpy as np
import pytest
import torch

import rank_bit_residual_b200 as rb
from synth import make_case
from tests.gpu_util import SyntheticWeight, assert_y_close, device, to_dev, x_tensor

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,M,N", [(1, 32, 16), (130, 160, 48), (257, 384, 272), (128, 1024, 512),
                                   (300, 3072, 3072)])
def test_int32_product_is_exact(B, M, N):
    rng = np.random.default_rng(B + M + N)
    w = SyntheticWeight(M, N, 0, "int8", seed=B)
    a = rng.integers(-127, 128, (B, M)).astype(np.int8)
    acc = rb.svdq_residual_product_i32(w.w, to_dev(a, torch.int8)).cpu().numpy()
    want = a.astype(np.int64) @ w.codes.astype(np.int64).T
    assert np.array_equal(acc.astype(np.int64), want), int((acc != want).sum())


@pytest.mark.parametrize("B", [1, 2, 64, 300])
def test_int32_product_is_exact_at_the_largest_k(B):
    # bits = 8 at K = 12288 (the large compute-bound shape): codes at +-127 make
    # |acc| reach 12288 * 127^2 = 198,193,152, the largest sum the INT grid
    # produces, below 2^31. B = 1, 2 run the GEMV path, 64 the split-K skinny
    # kernel, 300 the CTA-pair kernel.
    M, N = 12288, 3072
    rng = np.random.default_rng(B)
    w = SyntheticWeight(M, N, 0, "int8", seed=B)
    cw = rng.integers(-127, 128, (N, M)).astype(np.int8)
    cw[0], cw[1] = 127, -127
    cw[2] = np.where(np.arange(M) % 2 == 0, 127, -127)
    w.w.codes.copy_(torch.from_numpy(cw.view(np.uint8).reshape(-1)).to(w.w.codes.device))
    a = rng.integers(-127, 128, (B, M)).astype(np.int8)
    a[0] = 127
    if B > 1:
        a[1] = np.where(np.arange(M) % 2 == 0, -127, 127)
    acc = rb.svdq_residual_product_i32(w.w, to_dev(a, torch.int8)).cpu().numpy()
    want = a.astype(np.float64) @ cw.astype(np.float64).T    # exact: every sum is below 2^53
    assert acc[0, 0] == 127 * 127 * M and acc[0, 1] == -127 * 127 * M
    assert np.array_equal(acc.astype(np.float64), want), int((acc != want).sum())


CASES = [
    # B, M, N, rank, fmt, bias
    (16, 256, 128, 16, "int4", False),
    (1, 64, 16, 1, "int4", False),
    (37, 96, 48, 0, "int4", True),
    (130, 512, 272, 40, "int8", True),
    (256, 1024, 512, 128, "int4", False),
    (64, 512, 256, 256, "int2", True),
    (300, 3072, 768, 32, "int4", True),
]


@pytest.mark.parametrize("B,M,N,rank,fmt,bias", CASES)
@pytest.mark.parametrize("xdt", ["bf16", "f32"])
def test_linear_int_matches_oracle(B, M, N, rank, fmt, bias, xdt):
    wl = make_case(B, M, N, rank=rank, seed=B * 7 + N, dtype=xdt, bias=bias)
    w = SyntheticWeight(M, N, rank, fmt, seed=N + rank, scale=wl.scale)
    b = to_dev(wl.bias, torch.bfloat16) if bias else None
    y32 = rb.svdq_linear(w.w, x_tensor(wl), bias=b, out_dtype=torch.float32)
    y16 = rb.svdq_linear(w.w, x_tensor(wl), bias=b, out_dtype=torch.bfloat16)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    want = w.oracle_y(wl.x, wl.bias if bias else None)
    assert_y_close(y32.cpu().numpy(), want, f"{B}x{M}x{N} r={rank} {fmt} {xdt}")
    # bf16 output is the fp32 result rounded once (same arithmetic, last cast differs)
    assert torch.equal(y16, y32.to(torch.bfloat16))


def test_linear_strided_output_and_input():
    wl = make_case(40, 256, 64, rank=8, seed=11)
    w = SyntheticWeight(256, 64, 8, "int4", seed=2, scale=wl.scale)
    xbig = torch.zeros((40, 512), dtype=torch.bfloat16, device=device())
    xbig[:, :256] = x_tensor(wl)
    out = torch.full((40, 96), 7.0, dtype=torch.float32, device=device())
    y = rb.svdq_linear(w.w, xbig[:, :256], out=out[:, :64], out_dtype=torch.float32)
    assert torch.all(out[:, 64:] == 7.0)
    assert_y_close(y.cpu().numpy(), w.oracle_y(wl.x))


def test_linear_rejects_mismatched_input():
    w = SyntheticWeight(64, 32, 4, "int4", seed=0)
    with pytest.raises(ValueError):
        rb.svdq_linear(w.w, torch.zeros((3, 96), dtype=torch.bfloat16, device=device()))


NVFP4_CASES = [
    (16, 256, 128, 16, False),
    (1, 64, 16, 1, False),
    (37, 96, 48, 0, True),
    (130, 512, 272, 40, True),
    (256, 1024, 512, 128, False),
    (300, 3072, 768, 32, True),
]


@pytest.mark.parametrize("B,M,N,rank,bias", NVFP4_CASES)
@pytest.mark.parametrize("xdt", ["bf16", "f32"])
@pytest.mark.parametrize("given_gs", [False, True])
def test_linear_nvfp4_matches_oracle(B, M, N, rank, bias, xdt, given_gs):
    wl = make_case(B, M, N, rank=rank, seed=B * 5 + N, dtype=xdt, bias=bias)
    w = SyntheticWeight(M, N, rank, "nvfp4", seed=N + rank, scale=wl.scale)
    b = to_dev(wl.bias, torch.bfloat16) if bias else None
    gs = np.float32(321.0) if given_gs else None
    gs_t = to_dev(np.array([gs], np.float32), torch.float32) if given_gs else None
    y32 = rb.svdq_linear(w.w, x_tensor(wl), bias=b, out_dtype=torch.float32, act_global_scale=gs_t)
    y16 = rb.svdq_linear(w.w, x_tensor(wl), bias=b, out_dtype=torch.bfloat16, act_global_scale=gs_t)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    want = w.oracle_y(wl.x, wl.bias if bias else None, gs_x=gs)
    assert_y_close(y32.cpu().numpy(), want, f"nvfp4 {B}x{M}x{N} r={rank} {xdt}")
    assert torch.equal(y16, y32.to(torch.bfloat16))


@pytest.mark.parametrize("B,M,N,rank,bias", NVFP4_CASES + [(2048, 1152, 640, 32, True)])
@pytest.mark.parametrize("xdt", ["bf16", "f32"])
def test_linear_mxfp4_matches_oracle(B, M, N, rank, bias, xdt):
    wl = make_case(B, M, N, rank=rank, seed=B * 7 + N, dtype=xdt, bias=bias)
    w = SyntheticWeight(M, N, rank, "mxfp4", seed=N + 2 * rank, scale=wl.scale)
    b = to_dev(wl.bias, torch.bfloat16) if bias else None
    y32 = rb.svdq_linear(w.w, x_tensor(wl), bias=b, out_dtype=torch.float32)
    y16 = rb.svdq_linear(w.w, x_tensor(wl), bias=b, out_dtype=torch.bfloat16)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    want = w.oracle_y(wl.x, wl.bias if bias else None)
    assert_y_close(y32.cpu().numpy(), want, f"mxfp4 {B}x{M}x{N} r={rank} {xdt}")
    assert torch.equal(y16, y32.to(torch.bfloat16))


def test_linear_workspace_reused_across_shapes():
    """One workspace for calls of different batch sizes (the large- and the
    short-batch paths): each call equals a call on a fresh workspace, bit for
    bit, and the oracle within tolerance."""
    M, N, rank = 512, 256, 32
    w = SyntheticWeight(M, N, rank, "int4", seed=5)
    shared = rb.LinearWorkspace()
    for i, B in enumerate((300, 1024, 64, 300, 2048, 300)):
        wl = make_case(B, M, N, rank=0, seed=100 + i)
        x = x_tensor(wl)
        y_shared = rb.svdq_linear(w.w, x, out_dtype=torch.float32, workspace=shared)
        y_fresh = rb.svdq_linear(w.w, x, out_dtype=torch.float32, workspace=rb.LinearWorkspace())
        assert rb.svdq_check_status() == rb.SVDQ_OK
        assert torch.equal(y_shared, y_fresh), f"call {i} (B={B})"
        assert_y_close(y_shared.cpu().numpy(), w.oracle_y(wl.x), f"call {i} B={B}")


@pytest.mark.parametrize("B", [300, 2048])
@pytest.mark.parametrize("fmt", ["int4", "int8", "nvfp4", "mxfp4"])
def test_large_batch_linear_equals_separate_stages(B, fmt):
    """For B > 128, svdq_linear (activation pass, then the pair GEMM on the
    workspace's codes) must equal the two stages called one after the other
    through their own entry points, bit for bit, on repeated calls."""
    M, N, rank = 1536, 768, 32
    wl = make_case(B, M, N, rank=rank, seed=B + 1, bias=True)
    w = SyntheticWeight(M, N, rank, fmt, seed=3, scale=wl.scale)
    x = x_tensor(wl)
    scale = to_dev(wl.scale, torch.float32)
    b = to_dev(wl.bias, torch.bfloat16)
    gsw = w.w.w_scale if fmt == "nvfp4" else None
    codes, sf, s, down = rb.svdq_quantize_act(x, scale, fmt, ld=w.w.ld, w_global_scale=gsw)
    y_sep = rb.svdq_residual_linear(w.w, codes, sf, s, down, bias=b, out_dtype=torch.float32)
    for _ in range(5):
        y = rb.svdq_linear(w.w, x, bias=b, out_dtype=torch.float32)
        assert torch.equal(y, y_sep)
    assert rb.svdq_check_status() == rb.SVDQ_OK


@pytest.mark.parametrize("B", [1, 2, 3, 8, 16])
@pytest.mark.parametrize("M,N,rank,fmt,packed,bias,xdt", [
    (4096, 4096, 32, "int4", True, False, "bf16"),
    (3072, 3072, 128, "int8", False, True, "bf16"),
    (1056, 2000, 48, "int4", True, False, "f32"),
    (1024, 272, 16, "int4", False, True, "bf16"),
    (512, 48, 0, "int8", False, False, "f32"),
    (2048, 1040, 256, "int4", True, True, "f32"),
    (96, 16, 1, "int2", False, True, "bf16"),
])
def test_single_launch_decode_matches_oracle(B, M, N, rank, fmt, packed, bias, xdt):
    """Up to 16 rows with INT weights run as one kernel (maximum, down-projection and
    codes split over a cluster, dp4a dot products and epilogue): Y matches the oracle,
    and the staged entry points agree within the same tolerance."""
    wl = make_case(B, M, N, rank=rank, seed=B * 11 + M + N, dtype=xdt, bias=bias)
    w = SyntheticWeight(M, N, rank, fmt, seed=N + rank + 3, scale=wl.scale, packed=packed)
    b = to_dev(wl.bias, torch.bfloat16) if bias else None
    x = x_tensor(wl)
    y32 = rb.svdq_linear(w.w, x, bias=b, out_dtype=torch.float32)
    y16 = rb.svdq_linear(w.w, x, bias=b, out_dtype=torch.bfloat16)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    want = w.oracle_y(wl.x, wl.bias if bias else None)
    assert_y_close(y32.cpu().numpy(), want, f"decode B={B} {M}x{N} r={rank} {fmt}")
    assert torch.equal(y16, y32.to(torch.bfloat16))
    scale = to_dev(wl.scale, torch.float32)
    ld = w.w.ld if xdt == "bf16" else w.w.ld32
    codes, sf, s, down = rb.svdq_quantize_act(x, scale, fmt, ld=ld if rank else None)
    y_st = rb.svdq_residual_linear(w.w, codes, sf, s, down, bias=b, out_dtype=torch.float32)
    assert_y_close(y32.cpu().numpy(), y_st.cpu().numpy().astype(np.float64), "fused vs staged")


@pytest.mark.parametrize("B,N", [(300, 768), (520, 1280)])
def test_pair_split_tiles_equal_unsplit(B, N):
    """With a long K and fewer tiles than CTA pairs, svdq_linear cuts the tiles
    along K over several pairs (slice partials added by the owner, int32) while
    svdq_residual_linear (no workspace) does not split: the outputs are equal bit
    for bit, and match the oracle."""
    M, rank = 12288, 32
    wl = make_case(B, M, N, rank=rank, seed=B + N, bias=True)
    w = SyntheticWeight(M, N, rank, "int4", seed=5, scale=wl.scale, packed=True)
    x = x_tensor(wl)
    scale = to_dev(wl.scale, torch.float32)
    b = to_dev(wl.bias, torch.bfloat16)
    codes, sf, s, down = rb.svdq_quantize_act(x, scale, "int4", ld=w.w.ld)
    for out_dtype in (torch.float32, torch.bfloat16):
        y_sep = rb.svdq_residual_linear(w.w, codes, sf, s, down, bias=b, out_dtype=out_dtype)
        for _ in range(3):
            y = rb.svdq_linear(w.w, x, bias=b, out_dtype=out_dtype)
            assert torch.equal(y, y_sep), out_dtype
    assert rb.svdq_check_status() == rb.SVDQ_OK
    y32 = rb.svdq_linear(w.w, x, bias=b, out_dtype=torch.float32)
    assert_y_close(y32.cpu().numpy(), w.oracle_y(wl.x, wl.bias), f"split {B}x{M}x{N}")
