"""svdq_quantize_act_noalloc against svdq_quantize_act.

The allocation-free entry point serves callers that cannot allocate device memory
on their request path (a runtime that owns all device memory and hands out no
allocator, a plugin interface of another engine): it takes no workspace and uses
a fixed scratch array inside the library. Here it must give the same results as
the workspace entry point, on two calls in a row (the shared array keeps the
previous call's contents, which must not leak into the next result). This file
sorts last so a stop-at-first-failure run has already run everything else.
"""

import numpy as np
import pytest
import torch

import rank_bit_residual_b200 as rb
from synth import make_case, to_bf16
from tests.gpu_util import device, to_dev, x_tensor

pytestmark = pytest.mark.gpu


def _ld(rank, M, seed, dtype):
    rp = (rank + 15) // 16 * 16
    rng = np.random.default_rng(seed)
    ld = np.zeros((rp, M), np.float32)
    ld[:rank] = to_bf16(rng.standard_normal((rank, M)).astype(np.float32) * 0.1)
    return to_dev(ld, dtype)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "mxfp4"])
def test_noalloc_matches_workspace_entry_point_twice(fmt):
    device()
    cases = [make_case(300, 1024, 16, rank=0, seed=21), make_case(77, 512, 16, rank=0, seed=22)]
    for call, wl in enumerate(cases):          # two calls in a row, different shapes and data
        x = x_tensor(wl)
        scale = to_dev(wl.scale, torch.float32)
        ld = _ld(40, wl.M, 3 + call, torch.bfloat16)
        want = rb.svdq_quantize_act(x, scale, fmt, ld=ld)
        got = rb.svdq_quantize_act_noalloc(x, scale, fmt, ld=ld)
        assert rb.svdq_check_status() == rb.SVDQ_OK
        assert torch.equal(got[0], want[0]), "codes differ"
        if fmt != "int4":
            assert torch.equal(got[1], want[1]), "block scales differ"
        assert torch.equal(got[2], want[2]), "per-tensor scale differs"
        # down: same fp32 products, the K-split sums may be ordered differently
        d_got = got[3].float().cpu().numpy().astype(np.float64)
        d_want = want[3].float().cpu().numpy().astype(np.float64)
        rp = d_got.shape[1] // 2
        g, w = d_got[:, :rp] + d_got[:, rp:], d_want[:, :rp] + d_want[:, rp:]
        assert np.linalg.norm(g - w) <= 2e-5 * np.linalg.norm(w)


def test_noalloc_refuses_shapes_beyond_its_array():
    x = torch.zeros((16384, 256), dtype=torch.bfloat16, device=device())
    ld = torch.zeros((256, 256), dtype=torch.bfloat16, device=device())
    with pytest.raises(rb.SvdqError) as e:
        rb.svdq_quantize_act_noalloc(x, torch.ones(256, device=device()), "int4", ld=ld)
    assert e.value.status == rb.SVDQ_EWORKSPACE


# Shapes whose default plan does not fit the fixed 8 MiB array, so the entry point
# must halve the K split (and, for the last one, leave the short-batch plan for the
# large-batch one because fewer, wider column chunks outgrow its shared memory):
#   B = 8192, M = 3072, rank_pad 128: large-batch plan, K split 2 -> 1
#   B = 128, M = 4096, rank_pad 256: short-batch plan, 128 column chunks -> 32
#   B = 128, M = 16384, rank_pad 256: short-batch chunks of 256 columns need more
#     than 200 KB of shared memory -> large-batch plan, K split 128 -> 32
@pytest.mark.parametrize("B,M,rank", [(8192, 3072, 128), (128, 4096, 256), (128, 16384, 256)])
@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_noalloc_reduces_the_k_split_to_fit(B, M, rank, fmt):
    device()
    wl = make_case(B, M, 16, rank=0, seed=B + M + rank)
    x = x_tensor(wl)
    scale = to_dev(wl.scale, torch.float32)
    ld = _ld(rank, M, rank, torch.bfloat16)
    for _ in range(2):
        want = rb.svdq_quantize_act(x, scale, fmt, ld=ld)
        got = rb.svdq_quantize_act_noalloc(x, scale, fmt, ld=ld)
        assert rb.svdq_check_status() == rb.SVDQ_OK
        assert torch.equal(got[0], want[0]), "codes differ"
        if fmt != "int4":
            assert torch.equal(got[1], want[1]), "block scales differ"
        assert torch.equal(got[2], want[2]), "per-tensor scale differs"
        d_got = got[3].float().cpu().numpy().astype(np.float64)
        d_want = want[3].float().cpu().numpy().astype(np.float64)
        rp = d_got.shape[1] // 2
        g, w = d_got[:, :rp] + d_got[:, rp:], d_want[:, :rp] + d_want[:, rp:]
        assert np.linalg.norm(g - w) <= 2e-5 * np.linalg.norm(w)


def test_noalloc_returns_the_same_status_as_the_workspace_entry_point():
    # a misaligned down factor: both entry points answer SVDQ_EINVAL
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device=device())
    buf = torch.zeros(16 * 64 + 8, dtype=torch.bfloat16, device=device())
    ld = buf[1:1 + 16 * 64].view(16, 64)
    for fn in (rb.svdq_quantize_act, rb.svdq_quantize_act_noalloc):
        with pytest.raises(ValueError):
            fn(x, torch.ones(64, device=device()), "int4", ld=ld)
