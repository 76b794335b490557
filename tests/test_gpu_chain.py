"""Consecutive linears chained with programmatic dependent launch
(svdq_linear_ex with SVDQ_LINEAR_PDL; the enable_pdl option of
"flashinfer.gemm.svdquant_linear", here across layers): each activation pass
starts while the previous GEMM runs and reads its output only after
griddepcontrol.wait. The chained result must equal unchained calls bit for bit,
on both batch paths, in every format, inside CUDA graphs too, and the last
layer must match the oracle evaluated on the unchained intermediate."""

import numpy as np
import pytest
import torch

import rank_bit_residual_b200 as rb
from synth import make_case
from tests.gpu_util import SyntheticWeight, assert_y_close, to_dev, x_tensor

pytestmark = pytest.mark.gpu


def _layers(D, rank, fmt, n, seed, packed=False):
    return [SyntheticWeight(D, D, rank, fmt, seed=seed + i, packed=packed) for i in range(n)]


@pytest.mark.parametrize("B,D", [(1, 512), (16, 1024), (128, 2048), (300, 1024), (2048, 512)])
@pytest.mark.parametrize("fmt,packed", [("int4", True), ("int8", False), ("nvfp4", False), ("mxfp4", False)])
def test_chain_equals_unchained_calls(B, D, fmt, packed):
    wl = make_case(B, D, D, rank=0, seed=B + D)
    layers = _layers(D, 32, fmt, 3, seed=B, packed=packed)
    ws = [l.w for l in layers]
    x = x_tensor(wl)
    want = rb.svdq_linear_chain(ws, x, pdl=False)
    got = rb.svdq_linear_chain(ws, x, pdl=True)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    assert torch.equal(got, want)


@pytest.mark.parametrize("B", [16, 300])
def test_chain_last_layer_matches_oracle(B):
    D = 1024
    wl = make_case(B, D, D, rank=0, seed=7)
    layers = _layers(D, 32, "int4", 2, seed=3, packed=True)
    x = x_tensor(wl)
    y1 = rb.svdq_linear(layers[0].w, x)
    y2 = rb.svdq_linear(layers[1].w, y1, pdl=True, out_dtype=torch.float32)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    x2 = y1.float().cpu().numpy()
    assert_y_close(y2.cpu().numpy(), layers[1].oracle_y(x2), f"chained layer 2, B={B}")


@pytest.mark.parametrize("B,fmt", [(16, "int4"), (128, "nvfp4"), (300, "int4"), (64, "mxfp4")])
def test_chain_in_a_cuda_graph(B, fmt):
    D = 1024
    wl = make_case(B, D, D, rank=0, seed=B)
    layers = _layers(D, 32, fmt, 4, seed=11, packed=fmt == "int4")
    ws = [l.w for l in layers]
    x = x_tensor(wl)
    outs = [torch.empty((B, D), dtype=torch.bfloat16, device=x.device) for _ in ws]
    work = rb.LinearWorkspace()
    want = rb.svdq_linear_chain(ws, x, pdl=False).clone()
    rb.svdq_linear_chain(ws, x, pdl=True, workspace=work, outs=outs)   # sizes the workspace
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            rb.svdq_linear_chain(ws, x, pdl=True, workspace=work, outs=outs)
    for o in outs:
        o.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert rb.svdq_check_status() == rb.SVDQ_OK
    assert torch.equal(outs[-1], want)


def test_chain_repeated_is_deterministic():
    B, D = 128, 2048
    wl = make_case(B, D, D, rank=0, seed=5)
    ws = [l.w for l in _layers(D, 32, "int4", 4, seed=21, packed=True)]
    x = x_tensor(wl)
    work = rb.LinearWorkspace()
    first = rb.svdq_linear_chain(ws, x, workspace=work)
    for _ in range(20):
        y = rb.svdq_linear_chain(ws, x, workspace=work)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    assert torch.equal(first, y)
