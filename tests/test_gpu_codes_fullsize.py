"""Codes at full workload sizes against the page's definition.

"SVDQuant Smoothing, Low-rank and Residual Quantization", Formula and
conventions item 3: q = clamp(round_half_even(z / s), -qmax, qmax) with
s = max|z| / qmax, z = X_hat = x / scale (item 1) for the activation and z = R
for the residual. Here the GPU's codes are compared with that definition
evaluated in float64, given the GPU's stored s: every disagreement must lie
within one fp32 ulp of a half-integer and there may be at most 1e-5 of them;
the counts are printed. The codes must also equal the oracle's exactly rounded
quotients (oracle.codes), element for element, and s must equal the oracle's
fp32 s bit for bit. The fp4 formats are compared with the oracle's block
quantisers (exact e2m1 rounding, the stated fp32 scalars).
"""

import numpy as np
import pytest
import torch

import rank_bit_residual_b200 as rb
from oracle import codes as ocodes
from oracle import mxfp4 as omx
from oracle import nvfp4 as onv
from synth import make_workload
from tests.gpu_util import TIE_FRACTION, to_dev, x_tensor

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

CHUNK = 512   # rows per float64 chunk on the host


def _definition_compare(x, scale, s, bits, got):
    """(mismatches vs the float64 definition, mismatches outside the 1-ulp band,
    mismatches vs the oracle's exact codes)."""
    qm = 2 ** (bits - 1) - 1
    sc64 = scale.astype(np.float64)
    n_def = n_far = n_exact = 0
    for r0 in range(0, x.shape[0], CHUNK):
        xc = x[r0:r0 + CHUNK]
        g = got[r0:r0 + CHUNK].astype(np.int64)
        q64 = np.clip(np.rint(xc.astype(np.float64) / sc64[None, :] / np.float64(s)), -qm, qm)
        diff = g != q64
        near = ocodes.near_tie_1ulp(xc, scale[None, :], s)
        n_def += int(diff.sum())
        n_far += int((diff & ~near).sum())
        qe, _, _ = ocodes.act_codes_int(xc, scale, bits, s=s)
        n_exact += int((g != qe).sum())
    return n_def, n_far, n_exact


INT_CASES = [
    ("dit_attn_4096x3072x3072_int4", None),
    ("decode_128x4096x4096_int4", 128),
    ("decode_128x4096x4096_int4", 16),
    ("decode_128x4096x4096_int4", 1),
    ("large_8192x12288x3072_int4_r32", None),
    ("large_8192x12288x3072_int8_r32", None),
]


@pytest.mark.parametrize("name,rows", INT_CASES)
def test_act_int_codes_match_the_definition(name, rows):
    wl = make_workload(name)
    if rows is not None:
        wl = wl.rows(rows)
    codes, _, s, _ = rb.svdq_quantize_act(x_tensor(wl), to_dev(wl.scale, torch.float32), f"int{wl.bits}")
    assert rb.svdq_check_status() == rb.SVDQ_OK
    s_gpu = np.float32(s.item())
    s_oracle = ocodes.int_scale_fp32(ocodes.act_max_fp32(wl.x, wl.scale), wl.bits)
    assert s_gpu == s_oracle, (s_gpu, s_oracle)
    got = codes.cpu().numpy()
    n_def, n_far, n_exact = _definition_compare(wl.x, wl.scale, s_gpu, wl.bits, got)
    print(f"\n{name} B={wl.B}: {got.size} codes, {n_def} differ from the float64 definition "
          f"({n_far} outside the 1-ulp band), {n_exact} differ from the exact quotients")
    assert n_far == 0
    assert n_def <= TIE_FRACTION * got.size
    assert n_exact == 0


FP4_CASES = [
    ("dit_mlp_4096x3072x12288_nvfp4", None),
    ("dit_mlp_4096x3072x12288_mxfp4", None),
    ("decode_128x4096x4096_nvfp4", 128),
    ("decode_128x4096x4096_mxfp4", 128),
    ("decode_128x4096x4096_nvfp4", 1),
    ("large_8192x12288x3072_nvfp4_r32", None),
    ("large_8192x12288x3072_mxfp4_r32", None),
]


@pytest.mark.parametrize("name,rows", FP4_CASES)
def test_act_fp4_codes_and_scales_match_the_oracle(name, rows):
    wl = make_workload(name)
    if rows is not None:
        wl = wl.rows(rows)
    B, M = wl.B, wl.M
    codes, sf, g, _ = rb.svdq_quantize_act(x_tensor(wl), to_dev(wl.scale, torch.float32), wl.fmt)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    blk = 16 if wl.fmt == "nvfp4" else 32
    got_c = onv.unpack_nibbles(codes.cpu().numpy())
    got_sf = onv.sf_unswizzle(sf.cpu().numpy(), B, M // blk)
    gs = None
    if wl.fmt == "nvfp4":
        gs = onv.global_scale(ocodes.act_max_fp32(wl.x, wl.scale), "fp32")
        assert np.float32(g.item()) == gs
    n_c = n_sf = 0
    for r0 in range(0, B, CHUNK):
        xc = wl.x[r0:r0 + CHUNK]
        if wl.fmt == "nvfp4":
            c_o, sf_o, _ = onv.quantize(xc, gs=gs, div=wl.scale)
        else:
            c_o, sf_o = omx.quantize(xc, div=wl.scale)
        n_c += int((got_c[r0:r0 + CHUNK] != c_o).sum())
        n_sf += int((got_sf[r0:r0 + CHUNK] != sf_o).sum())
    print(f"\n{name} B={B}: {got_c.size} codes, {n_c} differ; {got_sf.size} scales, {n_sf} differ")
    assert n_c == 0 and n_sf == 0


RESIDUAL_CASES = [
    ("dit_attn_4096x3072x3072_int4", "int4"),
    ("large_8192x12288x3072_int4_r32", "int4"),
    ("large_8192x12288x3072_int8_r32", "int8"),
    ("large_8192x12288x3072_nvfp4_r32", "nvfp4"),
    ("large_8192x12288x3072_mxfp4_r32", "mxfp4"),
]


@pytest.mark.parametrize("name,fmt", RESIDUAL_CASES)
def test_residual_codes_of_prepare_match_the_definition(name, fmt):
    # rank 0: svdq_prepare quantises the smoothed weight fl32(scale W) itself, so the
    # residual the codes are taken of is known exactly on the host
    wl = make_workload(name, rows=8)
    M, N = wl.M, wl.N
    w = rb.svdq_prepare(to_dev(wl.W, torch.bfloat16), to_dev(wl.scale, torch.float32), 0, fmt)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    ws32 = (wl.scale[:, None].astype(np.float32) * wl.W.astype(np.float32)).astype(np.float32)
    f = rb.parse_fmt(fmt)
    if f.kind == rb.KIND_INT:
        s_w = np.float32(w.w_scale[0].item())
        assert s_w == ocodes.int_scale_fp32(np.max(np.abs(ws32)), f.bits)
        got = w.codes.view(torch.int8).cpu().numpy().reshape(N, M)
        # K-major: row n of the codes is column n of the residual
        n_def, n_far, n_exact = _definition_compare(np.ascontiguousarray(ws32.T), np.ones(M, np.float32),
                                                    s_w, f.bits, got)
        print(f"\n{name} residual {fmt}: {got.size} codes, {n_def} differ from the float64 definition "
              f"({n_far} outside the 1-ulp band), {n_exact} differ from the exact quotients")
        assert n_far == 0 and n_def <= TIE_FRACTION * got.size and n_exact == 0
    else:
        blk = 16 if fmt == "nvfp4" else 32
        got_c = onv.unpack_nibbles(w.codes.cpu().numpy().reshape(N, M // 2))
        got_sf = onv.sf_unswizzle(w.sf.cpu().numpy(), N, M // blk)
        wt = np.ascontiguousarray(ws32.T)
        if fmt == "nvfp4":
            c_o, sf_o, gs = onv.quantize(wt)
            assert np.float32(w.w_scale[0].item()) == gs
        else:
            c_o, sf_o = omx.quantize(wt)
        n_c, n_sf = int((got_c != c_o).sum()), int((got_sf != sf_o).sum())
        print(f"\n{name} residual {fmt}: {n_c} of {got_c.size} codes and {n_sf} scales differ")
        assert n_c == 0 and n_sf == 0
