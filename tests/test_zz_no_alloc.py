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
