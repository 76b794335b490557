"""MXFP4 oracle against the format definition (OCP microscaling, read from the
"mxfp4" per-block MinMax configuration of the SVDQuant parameter configuration
guide): the E8M0 table, the block exponent, worked blocks and invariants."""

import numpy as np
import pytest

from oracle import mxfp4 as mx
from oracle import nvfp4 as nv


def test_e8m0_table():
    c = np.arange(256)
    v = mx.e8m0_decode(c)
    assert np.isnan(v[255])
    assert np.array_equal(v[:255], [2.0 ** (e - 127) for e in range(255)])


@pytest.mark.parametrize("amax,X", [(6.0, 0), (7.99, 0), (8.0, 1), (5.99, 0), (4.0, 0), (3.99, -1),
                                    (1.0, -2), (0.75, -3), (2.0 ** -100, -102), (2.0 ** 200, 127),
                                    (2.0 ** -140, -127), (0.0, -127)])
def test_block_exponent(amax, X):
    assert mx.block_exponent(amax) == X


def test_worked_blocks():
    z = np.zeros((3, 32))
    z[0, :4] = [6.0, -3.0, 0.5, 1.25]   # X = 0: exact except 1.25 -> 1 (tie to even)
    z[1, :3] = [7.0, 2.5, -0.2]         # X = 0: 7 clips to 6, 2.5 -> 2 (tie to even), -0.2 -> 0
    z[2, :2] = [1.0, 0.3]               # X = -2: 4 and 1.2 -> 1 (codes in units of 0.25)
    codes, sf = mx.quantize(z)
    assert sf.tolist() == [[127], [127], [125]]
    d = mx.dequantize(codes, sf)
    assert d[0, :4].tolist() == [6.0, -3.0, 0.5, 1.0]
    assert d[1, :3].tolist() == [6.0, 2.0, 0.0]
    assert d[2, :2].tolist() == [1.0, 0.25]
    assert not np.any(codes[1, 2] & 0x8)          # -0.2 rounds to +0
    assert np.all(d[:, 4:] == 0)


def test_scaling_by_powers_of_two():
    rng = np.random.default_rng(0)
    z = rng.standard_normal((8, 64))
    c0, s0 = mx.quantize(z)
    for k in (-5, 3, 20):
        c1, s1 = mx.quantize(z * 2.0 ** k)
        assert np.array_equal(c0, c1)
        assert np.array_equal(s1.astype(int), s0.astype(int) + k)


def test_grid_values_round_trip():
    rng = np.random.default_rng(1)
    grid = nv.e2m1_decode(np.arange(16))
    vals = rng.choice(grid, (4, 64))
    vals[:, ::32] = 6.0                             # every block's amax is 6: X = 0
    codes, sf = mx.quantize(vals * 2.0 ** -9)
    assert np.all(sf == 127 - 9)
    assert np.array_equal(mx.dequantize(codes, sf), vals * 2.0 ** -9)


def test_error_bound_and_product():
    rng = np.random.default_rng(2)
    z = rng.standard_normal((16, 128))
    codes, sf = mx.quantize(z)
    d = mx.dequantize(codes, sf)
    # rounding moves a value by at most half the coarsest spacing (2 2^X between 4
    # and 6); clipping an amax in [6 2^X, 8 2^X) to 6 2^X by less than 2 2^X
    scale = mx.e8m0_decode(sf)
    err = np.abs(d - z).reshape(16, 4, 32)
    assert np.all(err < 2.0 * scale[:, :, None])
    inner = np.abs(z).reshape(16, 4, 32) <= 6.0 * scale[:, :, None]
    assert np.all(err[inner] <= np.broadcast_to(scale[:, :, None], err.shape)[inner])
    w = rng.standard_normal((8, 128))
    wc, ws = mx.quantize(w)
    assert np.allclose(mx.product(codes, sf, wc, ws), d @ mx.dequantize(wc, ws).T, rtol=0, atol=1e-12)


def test_linear_on_representable_operands_is_the_plain_product():
    """Operands already on the MXFP4 grid quantise to themselves, so the two-branch
    linear is x Ld Lu + x W^T + bias, summed here element by element."""
    from oracle import prepared as oprep
    rng = np.random.default_rng(3)
    grid = nv.e2m1_decode(np.arange(16))

    def on_grid(rows, K):
        v = rng.choice(grid, (rows, K))
        v[:, ::32] = 6.0
        return v * np.repeat(2.0 ** rng.integers(-6, 4, (rows, K // 32)), 32, axis=1)

    B, M, N, r = 2, 64, 3, 2
    x, W = on_grid(B, M), on_grid(N, M)
    ld, lu = rng.standard_normal((M, r)), rng.standard_normal((r, N))
    bias = rng.standard_normal(N)
    ca, sa = mx.quantize(x)
    cw, sw = mx.quantize(W)
    y = oprep.linear_mxfp4(x, ld, lu, ca, sa, cw, sw, bias)
    for b in range(B):
        for n in range(N):
            res = sum(x[b, k] * W[n, k] for k in range(M))
            low = sum(sum(x[b, k] * ld[k, j] for k in range(M)) * lu[j, n] for j in range(r))
            assert abs(y[b, n] - (res + low + bias[n])) <= 1e-12 * (1 + abs(res) + abs(low))
