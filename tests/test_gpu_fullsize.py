"""Full-size parity: every measured workload, in the launch configuration the bench
times (svdq_prepare then svdq_linear), checked on sampled output rows against the
oracle evaluated on the GPU's prepared buffers, and the split against the optimal
(Eckart-Young) tail of the smoothed weight."""

import numpy as np
import pytest
import torch

import rank_bit_residual_b200 as rb
from oracle import codes as ocodes
from oracle import mxfp4 as omx
from oracle import nvfp4 as onv
from oracle import prepared as oprep
from oracle import svdquant as osq
from synth import make_workload
from tests.gpu_util import assert_y_close, to_dev, x_tensor

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

CASES = [
    ("dit_attn_4096x3072x3072_int4", None),
    ("dit_mlp_4096x3072x12288_nvfp4", None),
    ("dit_mlp_4096x3072x12288_mxfp4", None),
    ("decode_128x4096x4096_int4", 1),
    ("decode_128x4096x4096_int4", 16),
    ("decode_128x4096x4096_int4", 128),
    ("decode_128x4096x4096_nvfp4", 1),
    ("decode_128x4096x4096_nvfp4", 128),
    ("decode_128x4096x4096_mxfp4", 1),
    ("decode_128x4096x4096_mxfp4", 128),
    ("large_8192x12288x3072_int4_r32", None),
    ("large_8192x12288x3072_int4_r128", None),
    ("large_8192x12288x3072_int8_r32", None),
    ("large_8192x12288x3072_int8_r128", None),
    ("large_8192x12288x3072_nvfp4_r32", None),
    ("large_8192x12288x3072_nvfp4_r128", None),
    ("large_8192x12288x3072_mxfp4_r32", None),
    ("large_8192x12288x3072_mxfp4_r128", None),
]

_prepared = {}


def _prepare(wl):
    key = (wl.name, wl.fmt, wl.bits, wl.rank)
    if key not in _prepared:
        _prepared.clear()
        fmt = f"int{wl.bits}" if wl.fmt == "int" else wl.fmt
        W = to_dev(wl.W, torch.bfloat16)
        w = rb.svdq_prepare(W, to_dev(wl.scale, torch.float32), wl.rank, fmt, seed=0)
        _prepared[key] = w
    return _prepared[key]


@pytest.mark.parametrize("name,rows", CASES)
def test_fullsize_sampled_parity(name, rows):
    wl = make_workload(name)
    if rows is not None:
        wl = wl.rows(rows)
    B, M, N = wl.B, wl.M, wl.N
    w = _prepare(wl)
    b = to_dev(wl.bias, torch.bfloat16) if wl.bias is not None else None
    y = rb.svdq_linear(w, x_tensor(wl), bias=b, out_dtype=torch.float32)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    rp = w.rank_pad
    ld = w.ld.float().cpu().numpy()[:rp].T
    L2 = w.lu.float().cpu().numpy()[:, :rp].T
    sample = np.random.default_rng(7).choice(B, size=min(B, 64), replace=False)
    if wl.fmt == "int":
        q, s_x, _ = ocodes.act_codes_int(wl.x, wl.scale, wl.bits)
        cw = w.codes.view(torch.int8).cpu().numpy().reshape(N, M)
        want = oprep.linear_int(wl.x[sample], ld, L2, q[sample], s_x, cw,
                                float(w.w_scale[0].item()), wl.bias)
    elif wl.fmt == "mxfp4":
        ca, sa = omx.quantize(wl.x[sample], div=wl.scale)
        cw = onv.unpack_nibbles(w.codes.cpu().numpy().reshape(N, M // 2))
        sfw = onv.sf_unswizzle(w.sf.cpu().numpy(), N, M // 32)
        want = oprep.linear_mxfp4(wl.x[sample], ld, L2, ca, sa, cw, sfw, wl.bias)
    else:
        ca, sa, gx = onv.quantize(wl.x, div=wl.scale)
        cw = onv.unpack_nibbles(w.codes.cpu().numpy().reshape(N, M // 2))
        sfw = onv.sf_unswizzle(w.sf.cpu().numpy(), N, M // 16)
        want = oprep.linear_nvfp4(wl.x[sample], ld, L2, ca[sample], sa[sample], gx, cw, sfw,
                                  float(w.w_scale[0].item()), wl.bias)
    got = y[torch.from_numpy(sample).to(y.device)].cpu().numpy()
    assert_y_close(got, want, f"{name} B={B}")


@pytest.mark.parametrize("name", ["dit_attn_4096x3072x3072_int4", "decode_128x4096x4096_int4",
                                  "large_8192x12288x3072_int4_r128"])
def test_fullsize_split_within_one_percent(name):
    wl = make_workload(name, rows=8)
    w = _prepare(wl)
    rp = w.rank_pad
    s = wl.scale.astype(np.float64)
    ws = s[:, None] * wl.W.astype(np.float64)
    ld = w.ld.float().cpu().numpy()[:rp].astype(np.float64)
    lu = w.lu.float().cpu().numpy()[:, :rp].astype(np.float64)
    R = ws - (s[:, None] * ld.T) @ lu.T
    tail = osq.tail_norm(ws, wl.rank)
    assert np.linalg.norm(R) <= 1.01 * tail, (np.linalg.norm(R), tail)
