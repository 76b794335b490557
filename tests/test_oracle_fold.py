"""Pins for the diagonal-fold geometric program (oracle.fold): the dither-model
identity against a Monte Carlo of subtractive dither, the closed form of a fold's
error against the identity, optimality (isotropic case, local perturbations, a brute
force over two channels, the migration-scale grid) and the gauge's scale invariance.
"Contraction-Gauge Preconditioning for Quantized Matrix Multiplication", abstract."""

import numpy as np
import pytest

from oracle import fold as ofold


def _dither(z, delta, rng):
    u = rng.uniform(-0.5, 0.5, z.shape)
    return delta * np.round(z / delta + u) - delta * u


def test_dither_identity_matches_monte_carlo():
    rng = np.random.default_rng(0)
    A = rng.standard_normal((6, 5))
    B = rng.standard_normal((5, 4)) * 0.3
    da, db = 0.4, 0.15
    errs = []
    for _ in range(20000):
        d = _dither(A, da, rng) @ _dither(B, db, rng) - A @ B
        errs.append(np.sum(d * d))
    mc = np.mean(errs)
    want = ofold.dither_error(A, B, da * da / 12, db * db / 12)
    se = np.std(errs) / np.sqrt(len(errs))
    assert abs(mc - want) <= 4 * se, (mc, want, se)


def test_fold_error_is_the_identity_on_the_folded_operands():
    rng = np.random.default_rng(1)
    x = rng.standard_t(3, (7, 9))
    W = rng.standard_normal((9, 5)) * 0.1
    t = rng.uniform(0.3, 3.0, 9)
    bits = 4
    q = 7.0
    A, B = x * t[None, :], W / t[:, None]
    da, db = np.max(np.abs(A)) / q, np.max(np.abs(B)) / q
    want = ofold.dither_error(A, B, da * da / 12, db * db / 12)
    got = ofold.fold_error(ofold.channel_stats(x, W), t, 7, 5, bits)
    assert got == pytest.approx(want, rel=1e-12)


def test_scale_invariance():
    rng = np.random.default_rng(2)
    st = ofold.channel_stats(rng.standard_normal((8, 6)), rng.standard_normal((6, 4)))
    t = rng.uniform(0.5, 2.0, 6)
    assert ofold.fold_error(st, 3.7 * t, 8, 4, 4) == pytest.approx(ofold.fold_error(st, t, 8, 4, 4), rel=1e-12)


def test_isotropic_channels_take_the_identity_fold():
    K = 8
    st = (np.full(K, 2.0), np.full(K, 10.0), np.full(K, 0.5), np.full(K, 3.0))
    t = ofold.gp_fold(st, 16, 12, 4)
    assert np.max(t) / np.min(t) == pytest.approx(1.0, abs=1e-6)


def _small_case(seed, K=12):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(3, (64, K))
    x[:, 3] *= 30.0
    W = rng.standard_normal((K, 16)) * 0.05
    W[5] *= 8.0
    return x, W


@pytest.mark.parametrize("seed", [3, 4, 5])
def test_gp_fold_is_a_local_minimum(seed):
    x, W = _small_case(seed)
    st = ofold.channel_stats(x, W)
    t = ofold.gp_fold(st, 64, 16, 4)
    e0 = ofold.fold_error(st, t, 64, 16, 4)
    for k in range(len(t)):
        for f in (1.0 - 1e-3, 1.0 + 1e-3):
            tt = t.copy()
            tt[k] *= f
            assert ofold.fold_error(st, tt, 64, 16, 4) >= e0 * (1 - 1e-9)


@pytest.mark.parametrize("seed", [6, 7])
def test_gp_fold_beats_the_migration_grid_and_the_identity(seed):
    x, W = _small_case(seed)
    st = ofold.channel_stats(x, W)
    e_gp = ofold.fold_error(st, ofold.gp_fold(st, 64, 16, 4), 64, 16, 4)
    for alpha in np.linspace(0.0, 1.0, 21):
        assert e_gp <= ofold.fold_error(st, ofold.alpha_fold(st, alpha), 64, 16, 4) * (1 + 1e-9)
    assert e_gp <= ofold.fold_error(st, np.ones(len(st[0])), 64, 16, 4)


def test_two_channels_brute_force():
    # two channels: by scale invariance the fold is one ratio t1 / t2; a fine
    # logarithmic grid of ratios reaches the program's optimum
    st = (np.array([3.0, 0.2]), np.array([40.0, 0.5]), np.array([0.1, 1.0]), np.array([0.2, 4.0]))
    t = ofold.gp_fold(st, 32, 8, 4)
    e_gp = ofold.fold_error(st, t, 32, 8, 4)
    ratios = np.exp(np.linspace(np.log(1e-4), np.log(1e4), 200001))
    best = min(ofold.fold_error(st, np.array([r, 1.0]), 32, 8, 4) for r in ratios[::50])
    i = np.argmin([ofold.fold_error(st, np.array([r, 1.0]), 32, 8, 4) for r in ratios[::50]])
    fine = ratios[max(0, i * 50 - 100): i * 50 + 100]
    best = min(best, min(ofold.fold_error(st, np.array([r, 1.0]), 32, 8, 4) for r in fine))
    assert e_gp <= best * (1 + 1e-9) and e_gp >= best * (1 - 1e-6)


def test_channels_without_a_product_term_keep_the_optimum():
    x, W = _small_case(8)
    x[:, 2] = 0.0          # an input channel that is always zero
    W[7] = 0.0             # a weight row that is zero
    st = ofold.channel_stats(x, W)
    t = ofold.gp_fold(st, 64, 16, 4)
    live = (st[0] > 0) & (st[2] > 0)
    a, _, b, _ = st
    assert np.max(a * t) == pytest.approx(1.0, rel=1e-9)                 # U = 1 kept
    assert np.max(b / t) == pytest.approx(np.max(b[live] / t[live]), rel=1e-9)   # V unchanged
