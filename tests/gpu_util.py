"""Helpers shared by the GPU tests: uploads, synthetic prepared weights, error metrics.

Expected values always come from the oracle package; the CUDA library is only
ever the thing under test.
"""

from __future__ import annotations

import numpy as np
import torch

import rank_bit_residual_b200 as rb
from oracle import codes as ocodes
from oracle import mxfp4 as omx
from oracle import nvfp4 as onv
from oracle import prepared as oprep
from synth import to_bf16

# Y tolerance of the operator (relative Frobenius and max-abs relative to max|Y|)
Y_REL_FRO = 2e-3
Y_MAX_REL = 1e-2
# near-tie code mismatches allowed, as a fraction of all elements
TIE_FRACTION = 1e-5


def device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


def to_dev(a: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    t = torch.from_numpy(a if a.flags.writeable else a.copy())
    return t.to(dtype).to(device())


def x_tensor(wl) -> torch.Tensor:
    return to_dev(wl.x, torch.bfloat16 if wl.x_dtype == "bf16" else torch.float32)


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64); b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_rel(a, b) -> float:
    a = np.asarray(a, np.float64); b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def assert_y_close(y_gpu, y_ref, what=""):
    rf, mr = rel_fro(y_gpu, y_ref), max_rel(y_gpu, y_ref)
    assert rf <= Y_REL_FRO and mr <= Y_MAX_REL, f"{what}: rel_fro={rf:.3e} max_rel={mr:.3e}"
    return rf, mr


def assert_codes_match(got: np.ndarray, want: np.ndarray, near: np.ndarray, what=""):
    mism = got.astype(np.int64) != want.astype(np.int64)
    n = int(mism.sum())
    assert np.all(near[mism]), f"{what}: {n} code mismatches, some not at a near-tie"
    assert n <= TIE_FRACTION * mism.size, f"{what}: {n} near-tie mismatches of {mism.size}"
    return n


class SyntheticWeight:
    """A prepared weight with random codes and factors (host copies kept for the oracle)."""

    def __init__(self, M, N, rank, fmt="int4", seed=0, scale=None, s_w=0.013, packed=False):
        rng = np.random.default_rng(seed)
        f = rb.parse_fmt(fmt)
        self.fmt, self.M, self.N, self.rank = f, M, N, rank
        self.rp = (rank + 15) // 16 * 16
        self.scale = scale if scale is not None else rng.uniform(0.5, 2.0, M).astype(np.float32)
        ld = np.zeros((max(self.rp, 1), M), np.float32)
        L2 = np.zeros((max(self.rp, 1), N), np.float32)
        if rank:
            ld[:rank] = to_bf16(rng.standard_normal((rank, M)).astype(np.float32) * 0.05)
            L2[:rank] = to_bf16(rng.standard_normal((rank, N)).astype(np.float32) / np.sqrt(N) * 4)
        self.ld = ld                                   # [rp, M]
        self.L2 = L2                                   # [rp, N]
        lu = np.zeros((N, max(2 * self.rp, 1)), np.float32)
        if self.rp:
            lu[:, :self.rp] = L2[:self.rp].T
            lu[:, self.rp:] = L2[:self.rp].T
        dev = device()
        if f.kind == rb.KIND_INT:
            qm = 2 ** (f.bits - 1) - 1
            self.codes = rng.integers(-qm, qm + 1, (N, M)).astype(np.int8)
            codes_buf = to_dev(self.codes.view(np.uint8).reshape(-1), torch.uint8)
            self.s_w = np.float32(s_w)
            sf_buf = None
            # the half-size copy the short-batch GEMM streams (nibble packing done here)
            codes4 = to_dev(onv.pack_nibbles(self.codes.view(np.uint8) & 0xF).reshape(-1),
                            torch.uint8) if packed else None
        elif f.kind == rb.KIND_MXFP4:
            self.codes = rng.integers(0, 16, (N, M)).astype(np.uint8)
            self.sf = rng.integers(121, 127, (N, M // 32)).astype(np.uint8)    # 2^-6 .. 2^-1
            codes_buf = to_dev(onv.pack_nibbles(self.codes).reshape(-1), torch.uint8)
            sf_buf = to_dev(onv.sf_swizzle(self.sf), torch.uint8)
            self.s_w = np.float32(1.0)
            codes4 = None
        else:
            self.codes = rng.integers(0, 16, (N, M)).astype(np.uint8)
            self.sf = rng.integers(0x20, 0x48, (N, M // 16)).astype(np.uint8)  # ~2^-3 .. 2^2
            codes_buf = to_dev(onv.pack_nibbles(self.codes).reshape(-1), torch.uint8)
            sf_buf = to_dev(onv.sf_swizzle(self.sf), torch.uint8)
            self.s_w = np.float32(2688.0 / 3.0)
            codes4 = None
        self.w = rb.weight_from_buffers(
            M, N, rank, f, codes_buf, sf_buf, to_dev(np.array([self.s_w], np.float32), torch.float32),
            to_dev(ld, torch.bfloat16), to_dev(ld, torch.float32), to_dev(lu, torch.bfloat16),
            to_dev(self.scale, torch.float32), codes4=codes4)

    def oracle_y(self, x: np.ndarray, bias=None, gs_x=None) -> np.ndarray:
        ldT = self.ld[: self.rp].T if self.rp else np.zeros((self.M, 0))
        L2 = self.L2[: self.rp] if self.rp else np.zeros((0, self.N))
        if self.fmt.kind == rb.KIND_INT:
            q, s_x, _ = ocodes.act_codes_int(x, self.scale, self.fmt.bits)
            return oprep.linear_int(x, ldT, L2, q, s_x, self.codes, self.s_w, bias)
        if self.fmt.kind == rb.KIND_MXFP4:
            ca, sa = omx.quantize(x, div=self.scale)
            return oprep.linear_mxfp4(x, ldT, L2, ca, sa, self.codes, self.sf, bias)
        ca, sa, gx = onv.quantize(x, gs=gs_x, div=self.scale)
        return oprep.linear_nvfp4(x, ldT, L2, ca, sa, gx, self.codes, self.sf, self.s_w, bias)
