"""svdq_fold_scale on the GPU against the oracle's geometric program (oracle.fold):
the GPU fold reaches the program's optimum (its dither-model error is the
oracle's, and no larger than that of any migration strength or the identity), and
it is a local minimum at the DiT attention shape where the oracle's generic solver
is too slow to run. "Contraction-Gauge Preconditioning for Quantized Matrix
Multiplication", abstract."""

import numpy as np
import pytest
import torch

import rank_bit_residual_b200 as rb
from oracle import fold as ofold
from synth import make_case, make_workload
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu


def _fold(x, W, bits, dt=torch.bfloat16):
    s = rb.svdq_fold_scale(to_dev(x, dt), to_dev(W, dt), bits)
    assert rb.svdq_check_status() == rb.SVDQ_OK
    return 1.0 / s.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("B,M,N,bits,dtype", [(512, 128, 96, 4, "bf16"), (300, 256, 64, 8, "f32"),
                                              (64, 96, 160, 4, "bf16")])
def test_fold_reaches_the_programs_optimum(B, M, N, bits, dtype):
    wl = make_case(B, M, N, rank=0, seed=B + M, dtype=dtype)
    t = _fold(wl.x, wl.W, bits, torch.bfloat16 if dtype == "bf16" else torch.float32)
    st = ofold.channel_stats(wl.x, wl.W)
    e_gpu = ofold.fold_error(st, t, B, N, bits)
    t_o = ofold.gp_fold(st, B, N, bits)
    e_o = ofold.fold_error(st, t_o, B, N, bits)
    assert e_gpu <= e_o * (1 + 1e-7) and e_gpu >= e_o * (1 - 1e-4), (e_gpu, e_o)
    a = st[0]
    tn, ton = t / np.max(a * t), t_o / np.max(a * t_o)
    assert np.max(np.abs(np.log(tn / ton))) <= 2e-3
    for alpha in (0.0, 0.25, 0.5, 0.75, 1.0):
        assert e_gpu <= ofold.fold_error(st, ofold.alpha_fold(st, alpha), B, N, bits) * (1 + 1e-7)


def test_fold_with_channels_without_a_product_term():
    wl = make_case(128, 64, 32, rank=0, seed=3, dtype="f32")
    x, W = wl.x.copy(), wl.W.copy()
    x[:, 5] = 0.0
    W[9] = 0.0
    t = _fold(x, W, 4, torch.float32)
    st = ofold.channel_stats(x, W)
    t_o = ofold.gp_fold(st, 128, 32, 4)
    assert ofold.fold_error(st, t, 128, 32, 4) <= ofold.fold_error(st, t_o, 128, 32, 4) * (1 + 1e-7)
    assert np.all(np.isfinite(t)) and np.all(t > 0)


def test_fold_is_a_local_minimum_at_full_size():
    wl = make_workload("dit_attn_4096x3072x3072_int4")
    t = _fold(wl.x, wl.W, 4)
    st = ofold.channel_stats(wl.x, wl.W)
    B, N = wl.B, wl.N
    e0 = ofold.fold_error(st, t, B, N, 4)
    rng = np.random.default_rng(0)
    for k in rng.choice(wl.M, 64, replace=False):
        for f in (1 - 1e-3, 1 + 1e-3):
            tt = t.copy()
            tt[k] *= f
            assert ofold.fold_error(st, tt, B, N, 4) >= e0 * (1 - 1e-9)
    for alpha in (0.25, 0.5, 0.75, 0.9):
        assert e0 <= ofold.fold_error(st, ofold.alpha_fold(st, alpha), B, N, 4)


def test_fold_vs_alpha_runs_the_two_branch_linear():
    from rank_bit_residual_b200.ablation import fold_vs_alpha
    wl = make_case(256, 256, 128, rank=0, seed=12, spikes=(4.0, 2.0))
    x = to_dev(wl.x, torch.bfloat16)
    W = to_dev(wl.W, torch.bfloat16)
    res = fold_vs_alpha(x, W, [0, 8], "int4", (0.5,), 4)
    assert set(res) == {"fold", "alpha=0.5"}
    for errs in res.values():
        assert all(0.0 < e < 1.0 for e in errs.values())
        assert errs[8] <= errs[0]
