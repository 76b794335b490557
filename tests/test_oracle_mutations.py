"""The pins catch plausible oracle mistakes: each case plants one in the oracle (CPU only)
and checks that at least one pin then fails."""

import numpy as np
import pytest

import oracle.svdquant as sq
import oracle.nvfp4 as nv
import oracle.prepared as pp
import oracle.codes as oc
import oracle.fold as of
from tests import test_oracle_fold as T6
from tests import test_oracle_svdquant as T1
from tests import test_oracle_codes as T2


def _golden_loader():
    import json, os
    root = os.path.join(os.path.dirname(__file__), "golden")
    return lambda n: json.load(open(os.path.join(root, n)))


def _fails(fn, *args):
    try:
        fn(*args)
    except (AssertionError, ValueError):
        return True
    return False


def _int_quantize_half_away(z, bits):
    z64 = np.array(z, dtype=np.float64)
    qm = sq.qmax_of(bits)
    s = float(np.max(np.abs(z64))) / qm if z64.size else 0.0
    if s == 0.0:
        return np.zeros(z64.shape, np.int64), 0.0
    t = z64 / s
    return np.clip(np.sign(t) * np.floor(np.abs(t) + 0.5), -qm, qm).astype(np.int64), s


def _int_quantize_wrong_qmax(z, bits):
    z64 = np.array(z, dtype=np.float64)
    qm = 2 ** (bits - 1)
    s = float(np.max(np.abs(z64))) / qm
    if s == 0.0:
        return np.zeros(z64.shape, np.int64), 0.0
    return np.clip(np.rint(z64 / s), -qm, qm).astype(np.int64), s


def _smooth_multiply(x, w, s):
    x64, w64, s64 = (np.array(a, dtype=np.float64) for a in (x, w, s))
    return x64 * s64[None, :], w64 / s64[:, None]


def _split_drop_sigma(weight, rank):
    sq.check_rank(weight, rank)
    w = np.array(weight, dtype=np.float64)
    if rank == 0:
        return np.zeros((w.shape[0], 0)), np.zeros((0, w.shape[1])), w.copy()
    U, S, Vt = np.linalg.svd(w, full_matrices=False)
    L, R = U[:, :rank], Vt[:rank]
    return L, R, w - L @ R


def _split_wrong_end(weight, rank):
    sq.check_rank(weight, rank)
    w = np.array(weight, dtype=np.float64)
    if rank == 0:
        return np.zeros((w.shape[0], 0)), np.zeros((0, w.shape[1])), w.copy()
    U, S, Vt = np.linalg.svd(w, full_matrices=False)
    L, R = U[:, -rank:] * S[-rank:], Vt[-rank:]
    return L, R, w - L @ R


def _linear_quantize_full_weight(x, weight, scale, rank, bits=4):
    sq.check_smoothing(x, weight, scale)
    xs, ws = sq.smooth_inputs(x, weight, scale)
    L1, L2, R = sq.split_weight(ws, rank)
    return (xs @ L1) @ L2 + sq.fake_quantize(xs, bits) @ sq.fake_quantize(ws, bits) - \
        (xs @ L1) @ L2 * 0


def _linear_quantized_low_rank(x, weight, scale, rank, bits=4):
    sq.check_smoothing(x, weight, scale)
    xs, ws = sq.smooth_inputs(x, weight, scale)
    L1, L2, R = sq.split_weight(ws, rank)
    qx = sq.fake_quantize(xs, bits)
    return (qx @ L1) @ L2 + qx @ sq.fake_quantize(R, bits)


def _e2m1_ties_away(v):
    v = np.asarray(v, dtype=np.float64)
    grid = nv._E2M1_GRID
    a = np.abs(v)
    idx = np.argmin(np.abs(a[..., None] - grid) - 1e-12 * np.arange(8), axis=-1)
    idx = np.where(a >= 6, 7, idx).astype(np.uint8)
    return (((v < 0) & (idx != 0)).astype(np.uint8) << 3) | idx


def _quotient_reciprocal_multiply(a, d1, d2):
    a32 = np.asarray(a, np.float32)
    c = ((np.float32(1) / np.asarray(d1, np.float32)).astype(np.float32) *
         np.float32(np.float32(1) / np.float32(d2))).astype(np.float32)
    return np.rint((a32 * c).astype(np.float32)).astype(np.float64)


def _quotient_two_divisions(a, d1, d2):
    a32 = np.asarray(a, np.float32)
    xs = (a32 / np.asarray(d1, np.float32)).astype(np.float32)
    return np.rint((xs / np.float32(d2)).astype(np.float32)).astype(np.float64)


def _quotient_half_away(a, d1, d2):
    t = np.asarray(a, np.float64) / (np.asarray(d1, np.float64) * np.float64(d2))
    return np.sign(t) * np.floor(np.abs(t) + 0.5)


def _e2m1_ratio_ties_away(p, c, negative):
    p = np.asarray(p, np.float64)
    c = np.broadcast_to(np.asarray(c, np.float64), p.shape)
    mids = 0.5 * (nv._E2M1_GRID[:-1] + nv._E2M1_GRID[1:])
    idx = np.zeros(p.shape, np.int64)
    for i, mid in enumerate(mids):
        idx = np.where(p >= mid * c, i + 1, idx)
    sign = (np.asarray(negative) & (idx != 0)).astype(np.uint8) << 3
    return (sign | idx.astype(np.uint8)).astype(np.uint8)


def _dither_error_no_cross(A, B, var_a, var_b):
    A = np.asarray(A, np.float64); B = np.asarray(B, np.float64)
    va = np.broadcast_to(np.asarray(var_a, np.float64), A.shape)
    vb = np.broadcast_to(np.asarray(var_b, np.float64), B.shape)
    return float(np.sum(va @ (B * B)) + np.sum((A * A) @ vb))


def _fold_error_delta_not_squared(stats, t, m, n, bits):
    a, alpha, b, beta = (np.asarray(s_, np.float64) for s_ in stats)
    q = float(2 ** (bits - 1) - 1)
    U, V = float(np.max(a * t)), float(np.max(b / t))
    return (m * U / (12 * q) * float(np.sum(beta / (t * t))) + n * V / (12 * q) * float(np.sum(alpha * t * t)) +
            len(a) * m * n * U * V / (144 * q * q))


def _pack_swapped(codes):
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 1::2] & 0xF) | ((c[:, 0::2] & 0xF) << 4)


def _sf_offset_transposed(r, c, rows, kblocks):
    _, kbp = nv.sf_padded_shape(rows, kblocks)
    r = np.asarray(r, dtype=np.int64); c = np.asarray(c, dtype=np.int64)
    atom = (r // 128) * (kbp // 4) + (c // 4)
    return atom * 512 + (r % 32) * 4 + ((r % 128) // 32) * 16 + (c % 4)


def _int_product_transposed(a, w):
    a = np.asarray(a, dtype=np.float64); w = np.asarray(w, dtype=np.float64)
    return a @ w[::-1].T


MUTATIONS = [
    (sq, "int_quantize", _int_quantize_half_away, [T1.test_fake_quantize_hand_cases]),
    (sq, "int_quantize", _int_quantize_wrong_qmax, [T1.test_fake_quantize_hand_cases]),
    (sq, "smooth_inputs", _smooth_multiply, [T1.test_svdquant_linear_hand_case]),
    (sq, "split_weight", _split_drop_sigma, [T1.test_split_weight_hand_case]),
    (sq, "split_weight", _split_wrong_end, [T1.test_split_weight_hand_case]),
    (sq, "svdquant_linear", _linear_quantize_full_weight, [T1.test_svdquant_linear_hand_case]),
    (sq, "svdquant_linear", _linear_quantized_low_rank, [T1.test_svdquant_linear_hand_case]),
    (nv, "e2m1_encode", _e2m1_ties_away, [T2.test_e2m1_rounding_ties]),
    (nv, "pack_nibbles", _pack_swapped, [T2.test_pack_nibbles_order]),
    (oc, "_exact_rne_quotient", _quotient_reciprocal_multiply,
     [T2.test_codes_decided_exactly_where_fp32_orders_differ]),
    (oc, "_exact_rne_quotient", _quotient_two_divisions,
     [T2.test_codes_decided_exactly_where_fp32_orders_differ]),
    (oc, "_exact_rne_quotient", _quotient_half_away, [T2.test_codes_hand_ties]),
    (nv, "e2m1_encode_ratio", _e2m1_ratio_ties_away, [T2.test_e2m1_ratio_ties_go_to_even]),
    (of, "dither_error", _dither_error_no_cross, [T6.test_dither_identity_matches_monte_carlo]),
    (of, "fold_error", _fold_error_delta_not_squared, [T6.test_fold_error_is_the_identity_on_the_folded_operands]),
    (nv, "sf_offset", _sf_offset_transposed, [T2.test_sf_layout_points_and_bijection]),
    (pp, "int_product", _int_product_transposed, [T1.test_integer_product_matches_brute_force]),
]


@pytest.mark.parametrize("mod,name,bad,pins", MUTATIONS,
                         ids=[f"{m[1]}:{m[2].__name__}" for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, mod, name, bad, pins):
    golden = _golden_loader()
    monkeypatch.setattr(mod, name, bad)
    caught = False
    for pin in pins:
        nargs = pin.__code__.co_argcount
        caught |= _fails(pin, golden) if nargs == 1 else _fails(pin)
    assert caught, f"no pin caught the planted mistake in {name}"


# ------------------------------------------------------------------ MXFP4
import oracle.mxfp4 as mx
from tests import test_oracle_mxfp4 as T5


@pytest.mark.parametrize("emax", [1, 3])
def test_mxfp4_wrong_element_exponent_is_caught(monkeypatch, emax):
    monkeypatch.setattr(mx, "E2M1_EMAX", emax)
    assert _fails(T5.test_worked_blocks) or _fails(T5.test_block_exponent, 6.0, 0)


def test_mxfp4_ceil_exponent_is_caught(monkeypatch):
    def ceil_exp(amax):
        a = np.asarray(amax, dtype=np.float64)
        x = np.ceil(np.log2(np.where(a > 0, a, 1.0))).astype(np.int64) - mx.E2M1_EMAX
        return np.where(a > 0, np.clip(x, -127, 127), -127)
    monkeypatch.setattr(mx, "block_exponent", ceil_exp)
    assert _fails(T5.test_worked_blocks)


def test_mxfp4_block_of_16_is_caught(monkeypatch):
    monkeypatch.setattr(mx, "BLOCK", 16)
    assert _fails(T5.test_worked_blocks) or _fails(T5.test_error_bound_and_product)
