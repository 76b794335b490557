"""Host check of the error bound behind the activation codes' near-half band.

The kernels estimate each INT code from x c_k, with c_k = fl(fl(1 / scale_k) u) and
u = fl(1 / s). They send an element to the exact re-decision when the distance of x c_k
to its rounded value exceeds 1/2 - 8 (qmax + 1) 2^-24. That is safe only if
|x c_k - x / (scale_k s)| < 3 (qmax + 1) 2^-24 for every element of the tensor.

Here that bound is measured with no GPU. The fp32 roundings of the constants are
numpy's, which are correctly rounded like the kernels'. x c_k is formed exactly in
float64: x has 24 significant bits and c_k has 24. The quotient x / (scale_k s) is
one float64 division, with a relative error of 2^-53, far below the bound. The
inputs are adversarial: scales over twenty binary orders, bf16 and fp32 x, and the
tensor maximum in every column.
"""

import numpy as np
import pytest

from oracle import codes as ocodes
from synth import to_bf16


def _estimate_error(x32, scale32, bits):
    s = ocodes.int_scale_fp32(ocodes.act_max_fp32(x32, scale32), bits)
    rk = (np.float32(1.0) / scale32).astype(np.float32)
    u = np.float32(np.float32(1.0) / s)
    ck = (rk * u).astype(np.float32)
    t = x32.astype(np.float64) * ck.astype(np.float64)[None, :]          # exact product
    q = x32.astype(np.float64) / (scale32.astype(np.float64)[None, :] * np.float64(s))
    return np.max(np.abs(t - q)), np.max(np.abs(q))


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_estimate_error_is_inside_the_band(bits, dtype, seed):
    rng = np.random.default_rng(100 * bits + seed)
    qm = ocodes.qmax_of(bits)
    B, M = 64, 512
    x = (rng.standard_normal((B, M)) * np.exp2(rng.integers(-6, 7, size=M))[None, :]).astype(np.float32)
    if dtype == "bf16":
        x = to_bf16(x)
    scale = np.exp2(rng.uniform(-10, 10, size=M)).astype(np.float32)
    # every column holds a value whose quotient is the tensor maximum
    amax = np.max(np.abs(x) / scale[None, :])
    x[0, :] = (amax * scale).astype(np.float32)
    if dtype == "bf16":
        x = to_bf16(x)
    err, qmax_seen = _estimate_error(x, scale, bits)
    bound = 3.0 * (qm + 1) * 2.0 ** -24
    band = 8.0 * (qm + 1) * 2.0 ** -24
    assert qmax_seen <= qm * (1 + 2.0 ** -23) + 1e-12
    assert err < bound, (err, bound)
    # the band covers the error plus the 2^-26 rounding of the distance
    assert err + 2.0 ** -26 < band


def test_a_narrower_band_would_not_be_safe():
    """The bound is not loose by orders of magnitude. Some element's error exceeds a
    hundredth of it, so a band sized from a much smaller error would let elements
    through on the wrong side of a half-integer."""
    rng = np.random.default_rng(5)
    qm = ocodes.qmax_of(8)
    x = rng.uniform(-1, 1, size=(256, 1024)).astype(np.float32)
    scale = np.exp2(rng.uniform(-10, 10, size=1024)).astype(np.float32)
    err, _ = _estimate_error(x, scale, 8)
    assert err > 0.01 * 3.0 * (qm + 1) * 2.0 ** -24
