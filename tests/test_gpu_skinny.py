"""Short-batch path (B <= 128) on the GPU against the oracle: the split-K cluster
GEMM with its distributed-shared-memory reduction, for every K split the launch
plan can pick, with the int8 and the packed 4-bit weight copy, and the packing
itself."""

import numpy as np
import pytest
import torch

import rank_bit_residual_b200 as rb
from oracle import nvfp4 as onv
from synth import make_case
from tests.gpu_util import SyntheticWeight, assert_y_close, to_dev, x_tensor

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,M", [(16, 64), (272, 1024), (3072, 256)])
def test_pack_int4_matches_nibble_packing(N, M):
    rng = np.random.default_rng(N + M)
    codes = rng.integers(-8, 8, (N, M)).astype(np.int8)
    got = rb.svdq_pack_int4(to_dev(codes, torch.int8)).cpu().numpy()
    want = onv.pack_nibbles(codes.view(np.uint8) & 0xF)
    assert np.array_equal(got, want)


# (B, M, N): cluster sizes 1..8 (K steps and tile count decide it), ragged N
# tiles, B from 1 to 128
SHAPES = [(1, 32, 16), (1, 4096, 4096), (16, 1024, 16), (77, 768, 272), (128, 4096, 3072),
          (128, 512, 12288), (33, 2048, 1040), (128, 128, 128), (5, 896, 144), (2, 512, 272)]


@pytest.mark.parametrize("B,M,N", SHAPES)
@pytest.mark.parametrize("packed", [False, True])
def test_short_batch_int32_product_is_exact(B, M, N, packed):
    rng = np.random.default_rng(B * 3 + M + N)
    w = SyntheticWeight(M, N, 0, "int4", seed=B + 1, packed=packed)
    a = rng.integers(-7, 8, (B, M)).astype(np.int8)
    acc = rb.svdq_residual_product_i32(w.w, to_dev(a, torch.int8)).cpu().numpy()
    want = a.astype(np.int64) @ w.codes.astype(np.int64).T
    assert np.array_equal(acc.astype(np.int64), want), int((acc != want).sum())


@pytest.mark.parametrize("B,M,N", SHAPES)
@pytest.mark.parametrize("fmt,packed", [("int4", True), ("int4", False), ("int8", False),
                                        ("nvfp4", False), ("mxfp4", False)])
def test_short_batch_linear_matches_oracle(B, M, N, fmt, packed):
    rank = 32 if M >= 64 and N >= 64 else 8
    wl = make_case(B, M, N, rank=rank, seed=B + 2 * N + M, bias=True)
    w = SyntheticWeight(M, N, rank, fmt, seed=N, scale=wl.scale, packed=packed)
    b = to_dev(wl.bias, torch.bfloat16)
    y = rb.svdq_linear(w.w, x_tensor(wl), bias=b, out_dtype=torch.float32)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    assert_y_close(y.cpu().numpy(), w.oracle_y(wl.x, wl.bias), f"{fmt} packed={packed} {B}x{M}x{N}")


@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "mxfp4"])
def test_chained_launch_equals_separate_calls(fmt):
    """svdq_linear launches the GEMM as a dependent launch of the activation pass
    (its weight loads overlap that kernel); the result must equal the two stages
    called one after the other, bit for bit."""
    B, M, N, rank = 64, 2048, 1024, 32
    wl = make_case(B, M, N, rank=rank, seed=5, bias=True)
    w = SyntheticWeight(M, N, rank, fmt, seed=9, scale=wl.scale, packed=fmt == "int4")
    x = x_tensor(wl)
    scale = to_dev(wl.scale, torch.float32)
    b = to_dev(wl.bias, torch.bfloat16)
    y1 = rb.svdq_linear(w.w, x, bias=b, out_dtype=torch.float32)
    gsw = w.w.w_scale if fmt == "nvfp4" else None
    codes, sf, s, down = rb.svdq_quantize_act(x, scale, fmt, ld=w.w.ld, w_global_scale=gsw)
    y2 = rb.svdq_residual_linear(w.w, codes, sf, s, down, bias=b, out_dtype=torch.float32)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    assert torch.equal(y1, y2)


def test_short_batch_repeated_calls_are_deterministic():
    B, M, N, rank = 128, 4096, 4096, 32
    wl = make_case(B, M, N, rank=rank, seed=3)
    w = SyntheticWeight(M, N, rank, "int4", seed=4, scale=wl.scale, packed=True)
    x = x_tensor(wl)
    ys = [rb.svdq_linear(w.w, x, out_dtype=torch.float32) for _ in range(3)]
    assert rb.svdq_check_status() == rb.SVDQ_OK
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])
