"""svdq_prepare and svdq_quantize_residual on the GPU against the oracle.

The randomized split is not unique, so it is gated the way the pages define a
good split: the residual of the stored factors must be within 1% of the
Eckart-Young optimum (the tail of the oracle's exact SVD). Codes are bit-exact
against the oracle's fp32 code mode for the same residual.
"""

import numpy as np
import pytest
import torch

import rank_bit_residual_b200 as rb
from oracle import codes as ocodes
from oracle import mxfp4 as omx
from oracle import nvfp4 as onv
from oracle import prepared as oprep
from oracle import svdquant as osq
from synth import make_case, make_workload, to_bf16
from tests.gpu_util import assert_codes_match, assert_y_close, device, to_dev, x_tensor

pytestmark = pytest.mark.gpu


def _host(w):
    rp = w.rank_pad
    ld = w.ld.float().cpu().numpy()[:rp].astype(np.float64)          # [rp, M]
    lu = w.lu.float().cpu().numpy().astype(np.float64)               # [N, 2 rp]
    return ld, lu


def _residual(wl, w):
    ld, lu = _host(w)
    rp = w.rank_pad
    s = wl.scale.astype(np.float64)
    ws = s[:, None] * wl.W.astype(np.float64)
    if rp == 0:
        return ws, ws
    return ws, ws - (s[:, None] * ld.T) @ lu[:, :rp].T


@pytest.mark.parametrize("M,N,rank,dtype", [(256, 128, 16, "f32"), (64, 512, 40, "bf16"),
                                            (512, 64, 64, "bf16"), (1024, 768, 32, "bf16"),
                                            (96, 96, 96, "f32"), (3072, 512, 128, "bf16"),
                                            (1024, 768, 200, "bf16")])
def test_prepare_residual_within_one_percent_of_optimal(M, N, rank, dtype):
    wl = make_case(8, M, N, rank=rank, seed=M + N, dtype=dtype, spikes=(6.0, 4.0, 3.0, 2.0, 1.0))
    W = to_dev(wl.W, torch.bfloat16 if dtype == "bf16" else torch.float32)
    w = rb.svdq_prepare(W, to_dev(wl.scale, torch.float32), rank, "int4", seed=1)
    ld, lu = _host(w)
    rp = w.rank_pad
    # layout: padded rows are zero, the up factor is stored twice, ld32 mirrors ld
    assert np.all(ld[rank:] == 0) and np.array_equal(lu[:, :rp], lu[:, rp:])
    assert np.array_equal(w.ld32.cpu().numpy()[:rp], w.ld.float().cpu().numpy()[:rp])
    ws, R = _residual(wl, w)
    tail = osq.tail_norm(ws, rank)
    nR = np.linalg.norm(R)
    if rank == min(M, N):
        # full rank: only the bf16 rounding of the stored factors is left
        assert nR <= 1e-2 * np.linalg.norm(ws), nR / np.linalg.norm(ws)
    else:
        assert nR <= 1.01 * tail, (nR, tail)


@pytest.mark.parametrize("fmt", ["int4", "int8", "int2"])
def test_prepare_rank_zero_quantises_smoothed_weight_exactly(fmt):
    wl = make_case(4, 256, 96, rank=0, seed=5)
    w = rb.svdq_prepare(to_dev(wl.W, torch.bfloat16), to_dev(wl.scale, torch.float32), 0, fmt)
    ws32 = (wl.scale[:, None].astype(np.float32) * wl.W.astype(np.float32)).astype(np.float32)
    bits = rb.parse_fmt(fmt).bits
    q, s, near = ocodes.residual_codes_int(ws32, bits)
    assert np.float32(w.w_scale[0].item()) == s
    got = w.codes.view(torch.int8).cpu().numpy().reshape(96, 256)
    assert_codes_match(got, q, near)


@pytest.mark.parametrize("M,N", [(32, 16), (256, 272), (1024, 3072)])
@pytest.mark.parametrize("fmt", ["int4", "int8", "nvfp4", "mxfp4"])
def test_quantize_residual_bit_exact(M, N, fmt):
    rng = np.random.default_rng(M + N)
    R = (rng.standard_t(4, (M, N)) * 0.02).astype(np.float32)
    codes, sf, g = rb.svdq_quantize_residual(to_dev(R, torch.float32), fmt)
    if fmt == "nvfp4":
        c_o, sf_o, g_o = onv.quantize(np.ascontiguousarray(R.T))
        assert np.float32(g.item()) == np.float32(g_o)
        assert np.array_equal(sf.cpu().numpy(), onv.sf_swizzle(sf_o))
        assert np.array_equal(onv.unpack_nibbles(codes.cpu().numpy()), c_o)
    elif fmt == "mxfp4":
        c_o, sf_o = omx.quantize(np.ascontiguousarray(R.T))
        assert g.item() == 1.0
        assert np.array_equal(sf.cpu().numpy(), onv.sf_swizzle(sf_o))
        assert np.array_equal(onv.unpack_nibbles(codes.cpu().numpy()), c_o)
    else:
        q, s, near = ocodes.residual_codes_int(R, rb.parse_fmt(fmt).bits)
        assert np.float32(g.item()) == s
        assert_codes_match(codes.cpu().numpy(), q, near)


@pytest.mark.parametrize("bad", [0.0, -1.0, float("nan"), float("inf")])
def test_prepare_rejects_bad_scale(bad):
    wl = make_case(4, 64, 32, rank=4, seed=1)
    s = wl.scale.copy()
    s[7] = bad
    with pytest.raises(ValueError):
        rb.svdq_prepare(to_dev(wl.W, torch.bfloat16), to_dev(s, torch.float32), 4, "int4")
    assert rb.svdq_check_status() == rb.SVDQ_OK


def test_prepare_then_linear_tiny_workload():
    wl = make_workload("tiny_16x256x128_int4")
    w = rb.svdq_prepare(to_dev(wl.W, torch.float32), to_dev(wl.scale, torch.float32), wl.rank, "int4")
    y = rb.svdq_linear(w, x_tensor(wl), out_dtype=torch.float32).cpu().numpy()
    ld, lu = _host(w)
    rp = w.rank_pad
    cw = w.codes.view(torch.int8).cpu().numpy().reshape(wl.N, wl.M)
    q, s_x, _ = ocodes.act_codes_int(wl.x, wl.scale, wl.bits)
    want = oprep.linear_int(wl.x, ld.T, lu[:, :rp].T, q, s_x, cw, float(w.w_scale[0].item()))
    assert_y_close(y, want, "tiny")
    # end to end against the unquantised product: the two-branch error stays small
    ref = wl.x.astype(np.float64) @ wl.W.astype(np.float64)
    e2e = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    naive = osq.fake_quantize(wl.x, 4) @ osq.fake_quantize(wl.W, 4)
    assert e2e < np.linalg.norm(naive - ref) / np.linalg.norm(ref)


def test_prepare_is_deterministic_for_a_seed():
    wl = make_case(4, 256, 128, rank=16, seed=9)
    W = to_dev(wl.W, torch.bfloat16); s = to_dev(wl.scale, torch.float32)
    a = rb.svdq_prepare(W, s, 16, "int4", seed=3)
    b = rb.svdq_prepare(W, s, 16, "int4", seed=3)
    assert torch.equal(a.codes, b.codes) and torch.equal(a.ld, b.ld) and torch.equal(a.lu, b.lu)


@pytest.mark.parametrize("M,N,rank,bias", [(256, 128, 16, False), (1024, 768, 32, True)])
def test_prepare_then_linear_nvfp4(M, N, rank, bias):
    wl = make_case(64, M, N, rank=rank, seed=M + 3, bias=bias)
    w = rb.svdq_prepare(to_dev(wl.W, torch.bfloat16), to_dev(wl.scale, torch.float32), rank, "nvfp4")
    b = to_dev(wl.bias, torch.bfloat16) if bias else None
    y = rb.svdq_linear(w, x_tensor(wl), bias=b, out_dtype=torch.float32).cpu().numpy()
    ld, lu = _host(w)
    rp = w.rank_pad
    cw = onv.unpack_nibbles(w.codes.cpu().numpy().reshape(N, M // 2))
    sfw = onv.sf_unswizzle(w.sf.cpu().numpy(), N, M // 16)
    gs_w = float(w.w_scale[0].item())
    ca, sa, gx = onv.quantize(wl.x, div=wl.scale)
    want = oprep.linear_nvfp4(wl.x, ld.T, lu[:, :rp].T, ca, sa, gx, cw, sfw, gs_w,
                              wl.bias if bias else None)
    assert_y_close(y, want, "prepare+nvfp4")
    # the residual codes are the oracle's NVFP4 codes of the GPU residual's own recipe
    ws, R = _residual(wl, w)
    assert np.linalg.norm(R) <= 1.01 * osq.tail_norm(ws, rank)


@pytest.mark.parametrize("M,N,rank,B", [(256, 128, 16, 64), (1024, 768, 32, 300)])
def test_prepare_then_linear_mxfp4(M, N, rank, B):
    wl = make_case(B, M, N, rank=rank, seed=M + 5, bias=True)
    w = rb.svdq_prepare(to_dev(wl.W, torch.bfloat16), to_dev(wl.scale, torch.float32), rank, "mxfp4")
    assert w.w_scale[0].item() == 1.0
    y = rb.svdq_linear(w, x_tensor(wl), bias=to_dev(wl.bias, torch.bfloat16), out_dtype=torch.float32)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    ld, lu = _host(w)
    rp = w.rank_pad
    cw = onv.unpack_nibbles(w.codes.cpu().numpy().reshape(N, M // 2))
    sfw = onv.sf_unswizzle(w.sf.cpu().numpy(), N, M // 32)
    ca, sa = omx.quantize(wl.x, div=wl.scale)
    want = oprep.linear_mxfp4(wl.x, ld.T, lu[:, :rp].T, ca, sa, cw, sfw, wl.bias)
    assert_y_close(y.cpu().numpy(), want, "prepare+mxfp4")
