"""Seeded generators for the SVDQuant linear workloads.

Each workload is the activation x[B,M], the weight W[M,N] (page-1 layout:
``x @ W``), a positive smoothing scale[M], an optional bias[N] and the
quantisation setting. Shapes and value distributions follow the workloads the
operator is measured on: diffusion-transformer attention / MLP projections and
LLM decode linears, with heavy-tailed activations that carry a few outlier
channels and weights made of a Gaussian bulk plus a handful of rank-1 spikes.

Draw order (fixed, NumPy ``Generator(PCG64(seed))``):
  1. x bulk [B, M]            (standard normal or Student-t)
  2. outlier channel indices  (a permutation of M, first k kept, sorted)
  3. W bulk [M, N]            (standard normal, times the bulk std)
  4. spike left vectors  [S, M]  (Gaussian, each normalised to unit length)
  5. spike right vectors [S, N]  (Gaussian, each normalised to unit length)
  6. bias [N]                 (only when the workload has one)
Outlier channels are multiplied by a constant factor, spikes are added as
sum_k sigma_k u_k v_k^T, then x and W are rounded to bf16 (RNE) when the
workload is a bf16 one. The smoothing scale is the usual SmoothQuant-style
migration recipe ``max|x_:,j|^a / max|W_j,:|^(1-a)`` computed from the rounded
tensors; the pages take smoothing scales as given, so this lives with the
inputs, not with the method.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np
import torch


def to_bf16(a: np.ndarray) -> np.ndarray:
    """Round a float array to bf16 (round-to-nearest-even); returned as float32."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Reinterpret raw bf16 bit patterns (uint16) as float32 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


@dataclass
class Workload:
    name: str
    x: np.ndarray                 # float32 [B, M]; bf16-representable when x_dtype == "bf16"
    x_dtype: str                  # "bf16" or "f32"
    W: np.ndarray                 # float32 [M, N]; bf16-representable when w_dtype == "bf16"
    w_dtype: str
    scale: np.ndarray             # float32 [M], > 0
    rank: int
    fmt: str                      # "int", "nvfp4" or "mxfp4"
    bits: int                     # 2..8 for "int", 4 for the fp4 formats
    bias: Optional[np.ndarray] = None   # float32 [N], bf16-representable
    seed: int = 0
    notes: dict = field(default_factory=dict)

    @property
    def B(self) -> int:
        return self.x.shape[0]

    @property
    def M(self) -> int:
        return self.x.shape[1]

    @property
    def N(self) -> int:
        return self.W.shape[1]

    def rows(self, n: int) -> "Workload":
        """The same workload restricted to the first n rows of x."""
        return Workload(self.name, self.x[:n], self.x_dtype, self.W, self.w_dtype,
                        self.scale, self.rank, self.fmt, self.bits, self.bias,
                        self.seed, dict(self.notes))


def _unit_rows(g: np.ndarray) -> np.ndarray:
    return g / np.linalg.norm(g, axis=1, keepdims=True)


def generate(B: int, M: int, N: int, *, seed: int, x_dist: str = "normal",
             t_dof: float = 3.0, dtype: str = "bf16",
             outlier_idx: Optional[Sequence[int]] = None,
             outlier_frac: float = 0.0, outlier_factor: float = 1.0,
             w_std: float = 0.02, spikes: Sequence[float] = (),
             alpha: float = 0.5, bias_std: Optional[float] = None):
    """Draw (x, W, scale, bias) with the fixed draw order in the module docstring."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if x_dist == "normal":
        x = rng.standard_normal((B, M), dtype=np.float64)
    elif x_dist == "student_t":
        x = rng.standard_t(t_dof, size=(B, M))
    else:
        raise ValueError(x_dist)
    if outlier_idx is None:
        k = int(round(outlier_frac * M))
        idx = np.sort(rng.permutation(M)[:k])
    else:
        idx = np.asarray(sorted(outlier_idx), dtype=np.int64)
    W = w_std * rng.standard_normal((M, N), dtype=np.float64)
    S = len(spikes)
    if S:
        U = _unit_rows(rng.standard_normal((S, M), dtype=np.float64))
        V = _unit_rows(rng.standard_normal((S, N), dtype=np.float64))
        W = W + (U.T * np.asarray(spikes, dtype=np.float64)[None, :]) @ V
    bias = None
    if bias_std is not None:
        bias = bias_std * rng.standard_normal(N, dtype=np.float64)
    x[:, idx] *= outlier_factor
    x = x.astype(np.float32)
    W = W.astype(np.float32)
    if dtype == "bf16":
        x = to_bf16(x)
        W = to_bf16(W)
    if bias is not None:
        bias = to_bf16(bias.astype(np.float32))
    xmax = np.max(np.abs(x.astype(np.float64)), axis=0)
    wmax = np.max(np.abs(W.astype(np.float64)), axis=1)
    xmax = np.where(xmax > 0, xmax, 1.0)
    wmax = np.where(wmax > 0, wmax, 1.0)
    scale = (xmax ** alpha / wmax ** (1.0 - alpha)).astype(np.float32)
    return x, W, scale, bias, idx


# name -> (generator kwargs, rank, fmt, bits); sizes follow the measured workloads.
_SPECS = {
    # tiny case the oracle finishes instantly: fp32, four x50 channels, 4 spikes
    "tiny_16x256x128_int4": dict(
        gen=dict(B=16, M=256, N=128, seed=0, x_dist="normal", dtype="f32",
                 outlier_idx=(3, 77, 140, 201), outlier_factor=50.0,
                 w_std=0.05, spikes=(4.0, 3.0, 2.0, 1.0), alpha=0.5),
        rank=16, fmt="int", bits=4),
    # DiT attention projection, INT4 per-tensor grid
    "dit_attn_4096x3072x3072_int4": dict(
        gen=dict(B=4096, M=3072, N=3072, seed=1, x_dist="student_t", dtype="bf16",
                 outlier_frac=0.01, outlier_factor=30.0, w_std=0.02,
                 spikes=tuple(np.linspace(5.0, 1.0, 8)), alpha=0.5),
        rank=32, fmt="int", bits=4),
    # DiT MLP up-projection, NVFP4, with bias
    "dit_mlp_4096x3072x12288_nvfp4": dict(
        gen=dict(B=4096, M=3072, N=12288, seed=2, x_dist="student_t", dtype="bf16",
                 outlier_frac=0.01, outlier_factor=30.0, w_std=0.02,
                 spikes=tuple(np.linspace(5.0, 1.0, 8)), alpha=0.5, bias_std=0.01),
        rank=32, fmt="nvfp4", bits=4),
    # LLM decode sweep (B = 1 / 16 / 128 take the first rows of this draw)
    "decode_128x4096x4096_int4": dict(
        gen=dict(B=128, M=4096, N=4096, seed=3, x_dist="normal", dtype="bf16",
                 outlier_frac=0.005, outlier_factor=20.0, w_std=0.02,
                 spikes=tuple(np.linspace(8.0, 0.5, 16)), alpha=0.5),
        rank=32, fmt="int", bits=4),
    "decode_128x4096x4096_nvfp4": dict(
        gen=dict(B=128, M=4096, N=4096, seed=3, x_dist="normal", dtype="bf16",
                 outlier_frac=0.005, outlier_factor=20.0, w_std=0.02,
                 spikes=tuple(np.linspace(8.0, 0.5, 16)), alpha=0.5),
        rank=32, fmt="nvfp4", bits=4),
    # the same two shapes with MXFP4 blocks (E8M0 scales per 32 elements)
    "dit_mlp_4096x3072x12288_mxfp4": dict(
        gen=dict(B=4096, M=3072, N=12288, seed=2, x_dist="student_t", dtype="bf16",
                 outlier_frac=0.01, outlier_factor=30.0, w_std=0.02,
                 spikes=tuple(np.linspace(5.0, 1.0, 8)), alpha=0.5, bias_std=0.01),
        rank=32, fmt="mxfp4", bits=4),
    "decode_128x4096x4096_mxfp4": dict(
        gen=dict(B=128, M=4096, N=4096, seed=3, x_dist="normal", dtype="bf16",
                 outlier_frac=0.005, outlier_factor=20.0, w_std=0.02,
                 spikes=tuple(np.linspace(8.0, 0.5, 16)), alpha=0.5),
        rank=32, fmt="mxfp4", bits=4),
    # large compute-bound sweep
    "large_8192x12288x3072_int4_r32": dict(
        gen=dict(B=8192, M=12288, N=3072, seed=4, x_dist="student_t", dtype="bf16",
                 outlier_frac=0.01, outlier_factor=30.0, w_std=0.02,
                 spikes=tuple(np.linspace(10.0, 0.3, 32)), alpha=0.5),
        rank=32, fmt="int", bits=4),
}
for _r in (32, 128):
    for _fmt, _bits in (("int", 4), ("int", 8), ("nvfp4", 4), ("mxfp4", 4)):
        _tag = f"{_fmt}{_bits}" if _fmt == "int" else _fmt
        _SPECS[f"large_8192x12288x3072_{_tag}_r{_r}"] = dict(
            gen=_SPECS["large_8192x12288x3072_int4_r32"]["gen"], rank=_r, fmt=_fmt, bits=_bits)

WORKLOADS = tuple(_SPECS)


_LAST_DRAW: dict = {}


def _draw(g: dict):
    """generate(**g), remembering the last draw: the workloads of one sweep share
    x, W and scale (only rank and format differ); callers must not modify them."""
    key = tuple(sorted((k, v if not isinstance(v, (list, tuple)) else tuple(v)) for k, v in g.items()))
    if key not in _LAST_DRAW:
        _LAST_DRAW.clear()
        _LAST_DRAW[key] = generate(**g)
    return _LAST_DRAW[key]


def make_workload(name: str, rows: Optional[int] = None) -> Workload:
    """Build a named workload; ``rows`` keeps only the first rows of x. Arrays are
    shared with the previous call of the same draw (treat them as read-only)."""
    spec = _SPECS[name]
    g = dict(spec["gen"])
    x, W, scale, bias, idx = _draw(g)
    wl = Workload(name=name, x=x, x_dtype=g["dtype"], W=W, w_dtype=g["dtype"],
                  scale=scale, rank=spec["rank"], fmt=spec["fmt"], bits=spec["bits"],
                  bias=bias, seed=g["seed"], notes={"outlier_idx": idx})
    return wl.rows(rows) if rows is not None else wl


def make_case(B: int, M: int, N: int, *, rank: int, fmt: str = "int", bits: int = 4,
              seed: int = 0, dtype: str = "bf16", bias: bool = False,
              spikes: Sequence[float] = (4.0, 2.0, 1.0), outlier_frac: float = 0.02,
              x_dist: str = "student_t") -> Workload:
    """A small workload of any shape, drawn with the same recipe (for ragged/edge tests)."""
    x, W, scale, b, idx = generate(B, M, N, seed=seed, x_dist=x_dist, dtype=dtype,
                                   outlier_frac=outlier_frac, outlier_factor=30.0,
                                   w_std=0.02, spikes=spikes, alpha=0.5,
                                   bias_std=0.01 if bias else None)
    return Workload(name=f"case_{B}x{M}x{N}", x=x, x_dtype=dtype, W=W, w_dtype=dtype,
                    scale=scale, rank=rank, fmt=fmt, bits=bits, bias=b, seed=seed,
                    notes={"outlier_idx": idx})
