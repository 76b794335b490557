"""Pins for the page-1 oracle (smoothing, SVD split, fake-quantize, two-branch linear).

Each pin comes from outside the oracle: values worked by hand from the
definitions on "SVDQuant Smoothing, Low-rank and Residual Quantization"
(tests/golden/*.json), closed forms (Eckart-Young through an eigenvalue
routine, a diagonal weight), brute force on tiny inputs, and invariants.
"""

import numpy as np
import pytest

from oracle import svdquant as sq
from oracle import prepared


def _rng(seed=0):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ validation
def test_check_smoothing_rejects_bad_layouts_and_scales():
    x = np.ones((3, 4)); w = np.ones((4, 5)); s = np.ones(4)
    sq.check_smoothing(x, w, s)
    bad = [
        (np.ones(4), w, s), (x, np.ones(4), s), (x, w, np.ones((4, 1))),
        (np.ones((0, 4)), w, s), (x, np.ones((4, 0)), s),
        (np.ones((3, 5)), w, s), (x, w, np.ones(3)),
        (x, w, np.array([1, 1, 0, 1.0])), (x, w, np.array([1, -1, 1, 1.0])),
        (x, w, np.array([1, np.nan, 1, 1.0])), (x, w, np.array([1, np.inf, 1, 1.0])),
    ]
    for args in bad:
        with pytest.raises(ValueError):
            sq.check_smoothing(*args)


def test_check_rank_rejects_non_ints_and_out_of_range():
    w = np.ones((4, 3))
    for r in (0, 1, 3):
        sq.check_rank(w, r)
    for r in (-1, 4, True, False, 1.0, np.int64(1), "1", None):
        with pytest.raises(ValueError):
            sq.check_rank(w, r)
    with pytest.raises(ValueError):
        sq.check_rank(np.ones((2, 2, 2)), 1)


# ------------------------------------------------------------------- smoothing
def test_smoothing_preserves_product_and_inputs():
    rng = _rng(1)
    x = rng.standard_normal((7, 9)); w = rng.standard_normal((9, 5))
    s = rng.uniform(0.1, 10.0, 9)
    x0, w0, s0 = x.copy(), w.copy(), s.copy()
    xs, ws = sq.smooth_inputs(x, w, s)
    np.testing.assert_allclose(xs @ ws, x @ w, rtol=1e-12, atol=1e-12)
    assert np.array_equal(x, x0) and np.array_equal(w, w0) and np.array_equal(s, s0)
    assert xs.shape == x.shape and ws.shape == w.shape


def test_smoothing_power_of_two_scale_is_bit_exact():
    rng = _rng(2)
    x = rng.standard_normal((5, 8)); w = rng.standard_normal((8, 3))
    s = 2.0 ** rng.integers(-6, 7, 8)
    xs, ws = sq.smooth_inputs(x, w, s)
    # scaling by 2^k is exact, so every product and sum is bit-identical
    assert np.array_equal(xs @ ws, x @ w)


def test_smoothing_accepts_strided_views():
    rng = _rng(3)
    big_x = rng.standard_normal((10, 16)); big_w = rng.standard_normal((16, 12))
    s = rng.uniform(0.5, 2.0, 16)
    xv = big_x[::2, :]; wv = big_w[:, ::3]
    xs, ws = sq.smooth_inputs(xv, wv, s)
    xs2, ws2 = sq.smooth_inputs(np.ascontiguousarray(xv), np.ascontiguousarray(wv), s)
    assert np.array_equal(xs, xs2) and np.array_equal(ws, ws2)


# -------------------------------------------------------------------- SVD split
def test_split_weight_hand_case(golden):
    g = golden("split_weight_4x3.json")
    W = np.array(g["weight"])
    for r, key in ((1, "residual_rank1"), (2, "residual_rank2")):
        L, R_, res = sq.split_weight(W, r)
        assert L.shape == (4, r) and R_.shape == (r, 3)
        np.testing.assert_allclose(res, np.array(g[key]), atol=1e-12)
        np.testing.assert_allclose(L @ R_ + res, W, atol=1e-12)
    for r in range(4):
        res = sq.split_weight(W, r)[2]
        assert abs(np.sum(res ** 2) - g["residual_norm_sq"][r]) < 1e-10


def test_split_weight_rank_zero_and_full():
    rng = _rng(4)
    W = rng.standard_normal((6, 4))
    L, R_, res = sq.split_weight(W, 0)
    assert L.shape == (6, 0) and R_.shape == (0, 4)
    assert np.array_equal(res, W)
    L, R_, res = sq.split_weight(W, 4)
    assert np.linalg.norm(res) <= 1e-13 * np.linalg.norm(W)


def test_split_weight_diagonal_closed_form():
    W = np.zeros((5, 4)); W[0, 0] = 2.0; W[1, 1] = -5.0; W[2, 2] = 1.0; W[3, 3] = 3.0
    L, R_, res = sq.split_weight(W, 2)
    keep = np.zeros_like(W); keep[1, 1] = -5.0; keep[3, 3] = 3.0
    np.testing.assert_allclose(L @ R_, keep, atol=1e-13)
    np.testing.assert_allclose(res, W - keep, atol=1e-13)


@pytest.mark.parametrize("shape,r", [((40, 25), 3), ((25, 40), 7), ((32, 32), 16)])
def test_split_weight_eckart_young_via_eigenvalues(shape, r):
    rng = _rng(5)
    W = rng.standard_normal(shape)
    res = sq.split_weight(W, r)[2]
    # eigenvalues of W^T W (a symmetric eigensolver, not the SVD) give sigma^2
    lam = np.sort(np.linalg.eigvalsh(W.T @ W if shape[0] >= shape[1] else W @ W.T))[::-1]
    lam = np.clip(lam, 0, None)
    assert abs(np.sum(res ** 2) - np.sum(lam[r:])) <= 1e-9 * np.sum(lam)
    # spectral norm of the residual by power iteration equals sigma_{r+1}
    v = rng.standard_normal(shape[1])
    for _ in range(3000):
        v = res.T @ (res @ v); v /= np.linalg.norm(v)
    assert abs(np.linalg.norm(res @ v) - np.sqrt(lam[r])) <= 1e-6 * np.sqrt(lam[0])


def test_split_weight_beats_random_rank_r_competitors():
    rng = _rng(6)
    W = rng.standard_normal((30, 20)) + 3.0 * np.outer(rng.standard_normal(30), rng.standard_normal(20))
    r = 4
    best = np.linalg.norm(sq.split_weight(W, r)[2])
    for _ in range(50):
        Q, _ = np.linalg.qr(rng.standard_normal((30, r)))
        assert np.linalg.norm(W - Q @ (Q.T @ W)) >= best - 1e-12


# ---------------------------------------------------------------- fake quantize
def test_fake_quantize_hand_cases(golden):
    for c in golden("fake_quantize_cases.json")["cases"]:
        q, s = sq.int_quantize(np.array(c["z"]), c["bits"])
        assert s == c["s"]
        assert q.tolist() == c["codes"]
        np.testing.assert_array_equal(sq.fake_quantize(np.array(c["z"]), c["bits"]), c["q"])


@pytest.mark.parametrize("bits", range(2, 9))
def test_fake_quantize_invariants(bits):
    rng = _rng(bits)
    z = rng.standard_t(3, (13, 17))
    qm = 2 ** (bits - 1) - 1
    codes, s = sq.int_quantize(z, bits)
    Q = sq.fake_quantize(z, bits)
    assert np.all(np.abs(codes) <= qm)
    assert np.max(np.abs(codes)) == qm                       # the max element hits the grid end
    assert np.all(np.abs(Q - z) <= s / 2 * (1 + 1e-12))      # within half a step
    np.testing.assert_array_equal(sq.fake_quantize(-z, bits), -Q)   # odd symmetry
    np.testing.assert_array_equal(sq.fake_quantize(4.0 * z, bits), 4.0 * Q)  # power-of-two scaling
    assert np.array_equal(sq.fake_quantize(np.zeros((3, 4)), bits), np.zeros((3, 4)))
    # brute force: the chosen code is the nearest grid point
    grid = np.arange(-qm, qm + 1) * s
    nearest = np.min(np.abs(z[..., None] - grid), axis=-1)
    assert np.all(np.abs(Q - z) <= nearest + 1e-12)


def test_fake_quantize_rejects_bad_bits():
    for b in (1, 9, 0, 4.0, True):
        with pytest.raises(ValueError):
            sq.fake_quantize(np.ones(3), b)


# ------------------------------------------------------------ two-branch linear
def test_svdquant_linear_hand_case(golden):
    g = golden("svdquant_linear_2x2.json")
    x, W, s = np.array(g["x"]), np.array(g["weight"]), np.array(g["scale"])
    np.testing.assert_allclose(sq.svdquant_linear(x, W, s, 1, bits=2), g["y_bits2"], atol=1e-12)
    np.testing.assert_allclose(sq.svdquant_linear(x, W, s, 1, bits=4), g["y_bits4"], atol=1e-12)
    xs, ws = sq.smooth_inputs(x, W, s)
    L, R_, res = sq.split_weight(ws, 1)
    np.testing.assert_allclose((xs @ L) @ R_, g["low_rank"], atol=1e-12)
    np.testing.assert_allclose(res, g["residual"], atol=1e-12)


def test_svdquant_linear_full_rank_recovers_product():
    rng = _rng(7)
    x = rng.standard_normal((6, 10)); W = rng.standard_normal((10, 8))
    s = rng.uniform(0.5, 2.0, 10)
    Y = sq.svdquant_linear(x, W, s, 8, bits=4)
    np.testing.assert_allclose(Y, x @ W, rtol=1e-10, atol=1e-10)


def test_svdquant_linear_error_shrinks_with_bits_and_rank():
    rng = _rng(8)
    x = rng.standard_normal((64, 48)); x[:, 5] *= 30.0
    W = 0.05 * rng.standard_normal((48, 40)) + 2.0 * np.outer(rng.standard_normal(48), rng.standard_normal(40)) / 40
    s = np.sqrt(np.max(np.abs(x), 0)) / np.sqrt(np.max(np.abs(W), 1))
    ref = x @ W
    err = {b: np.linalg.norm(sq.svdquant_linear(x, W, s, 4, bits=b) - ref) for b in (2, 4, 8)}
    assert err[8] < err[4] < err[2]
    e_r = [np.linalg.norm(sq.svdquant_linear(x, W, s, r, bits=4) - ref) for r in (0, 8, 48 - 8)]
    assert e_r[2] < e_r[0]


def test_svdquant_linear_validates_and_leaves_inputs():
    rng = _rng(9)
    x = rng.standard_normal((3, 4)); W = rng.standard_normal((4, 5)); s = np.ones(4)
    x0, W0 = x.copy(), W.copy()
    sq.svdquant_linear(x, W, s, 2)
    assert np.array_equal(x, x0) and np.array_equal(W, W0)
    with pytest.raises(ValueError):
        sq.svdquant_linear(x, W, s, 5)
    with pytest.raises(ValueError):
        sq.svdquant_linear(x, W, -s, 1)


# ------------------------------------------------------------- prepared linear
def test_prepared_int_linear_equals_page_definition():
    """The folded form x Ld Lu + s_x s_w C_x C_w^T is the page-1 equation."""
    rng = _rng(10)
    B, M, N, r, bits = 9, 24, 16, 3, 4
    x = rng.standard_normal((B, M)); W = rng.standard_normal((M, N)); s = rng.uniform(0.3, 3, M)
    xs, ws = sq.smooth_inputs(x, W, s)
    L1, L2, R = sq.split_weight(ws, r)
    cx, sx = sq.int_quantize(xs, bits)
    cw, sw = sq.int_quantize(R, bits)
    Ld = L1 / s[:, None]
    Y = prepared.linear_int(x, Ld, L2, cx, sx, cw.T, sw)
    np.testing.assert_allclose(Y, sq.svdquant_linear(x, W, s, r, bits), rtol=1e-12, atol=1e-12)


def test_integer_product_matches_brute_force():
    rng = _rng(11)
    a = rng.integers(-127, 128, (5, 37)); w = rng.integers(-127, 128, (6, 37))
    brute = [[sum(int(a[i, k]) * int(w[j, k]) for k in range(37)) for j in range(6)] for i in range(5)]
    assert prepared.int_product(a, w).astype(np.int64).tolist() == brute
    # the largest magnitude the kernels meet (K = 12288, 8-bit) stays exact in float64
    K = 12288
    big = prepared.int_product(np.full((1, K), 127), np.full((1, K), -127))
    assert big[0, 0] == -127 * 127 * K


def test_tail_norm_matches_split_residual():
    rng = _rng(12)
    for shape, r in (((50, 30), 5), ((30, 50), 0), ((40, 40), 40)):
        W = rng.standard_normal(shape)
        res = sq.split_weight(W, r)[2]
        assert abs(sq.tail_norm(W, r) - np.linalg.norm(res)) <= 1e-9 * np.linalg.norm(W)
