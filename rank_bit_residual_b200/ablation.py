"""Accuracy ablation of the SVDQuant linear, run through this library on the GPU.

"SVDQuant Smoothing, Low-rank and Residual Quantization", section "Toy experiment":
synthetic activations with a 30x channel, and the output errors and singular-value
curves of three ways to run a low-bit linear - quantising x and W directly (naive
W4A4), smoothing first (smoothing only), and smoothing plus the rank-r branch in
high precision (two-branch) - at ranks 0 to 6. Here every variant is one
svdq_prepare + svdq_linear of this library (the smoothing-only variant is the
two-branch one at rank 0; the naive one uses a scale of ones), the error is the
relative Frobenius distance of Y to x @ W (float64), and the singular values are those
of W and of the smoothed weight diag(scale) W, whose leading directions are what a
rank-r branch can keep out of the quantiser.

    python -m rank_bit_residual_b200.ablation [--workload NAME] [--rows B] [--ranks 0,1,2,...]

prints one JSON object (errors per variant and rank, singular values, timings).
"""

from __future__ import annotations

import argparse
import json
import os
import sys
import time
from typing import Dict, Optional, Sequence

import numpy as np
import torch

from . import svdq_linear, svdq_prepare


def rel_fro(y: torch.Tensor, ref: torch.Tensor) -> float:
    d = (y.double() - ref).norm().item()
    return d / ref.norm().item()


def singular_values(a: np.ndarray, k: int) -> np.ndarray:
    """The k largest singular values of a (float64, LAPACK on the host)."""
    return np.linalg.svd(np.asarray(a, dtype=np.float64), compute_uv=False)[:k]


def ablation(x: torch.Tensor, W: torch.Tensor, scale: torch.Tensor, ranks: Sequence[int] = tuple(range(7)),
             fmt: str = "int4", seed: int = 0, n_sigma: int = 16) -> Dict:
    """Errors of the three variants (two-branch at each rank) and the singular values.

    x [B, M] and W [M, N] on the GPU (bf16 or fp32), scale [M] fp32 (the smoothing
    scale). Returns a dict of plain numbers.
    """
    if x.dim() != 2 or W.dim() != 2 or x.shape[1] != W.shape[0] or scale.shape != (W.shape[0],):
        raise ValueError("x must be [B, M], W [M, N] and scale [M]")
    ref = x.double() @ W.double()
    out = {"B": x.shape[0], "M": W.shape[0], "N": W.shape[1], "fmt": fmt, "ranks": list(ranks)}
    timing = {}

    def run(sc, r):
        t0 = time.perf_counter()
        w = svdq_prepare(W, sc, r, fmt, seed=seed)
        t1 = time.perf_counter()
        y = svdq_linear(w, x, out_dtype=torch.float32)
        torch.cuda.synchronize()
        timing.setdefault("prepare_s", []).append(t1 - t0)
        return rel_fro(y, ref)

    out["naive"] = run(torch.ones_like(scale), 0)
    out["smooth_only"] = run(scale, 0)
    out["two_branch"] = {int(r): run(scale, int(r)) for r in ranks}
    Wn = W.double().cpu().numpy()
    sn = scale.double().cpu().numpy()
    out["sigma_W"] = singular_values(Wn, n_sigma).tolist()
    s_ws = singular_values(sn[:, None] * Wn, max(n_sigma, max(ranks) + 1))
    out["sigma_smoothed"] = s_ws[:n_sigma].tolist()
    # share of the smoothed weight's Frobenius norm that a rank-r branch keeps out of the quantiser
    fro2 = float(np.sum((sn[:, None] * Wn) ** 2))
    out["kept_energy"] = {int(r): float(np.sum(s_ws[:r] ** 2) / fro2) for r in ranks}
    out["prepare_s_median"] = float(np.median(timing["prepare_s"]))
    return out


def main(argv: Optional[Sequence[str]] = None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="dit_attn_4096x3072x3072_int4")
    ap.add_argument("--rows", type=int, default=None, help="keep only the first rows of x")
    ap.add_argument("--ranks", default="0,1,2,3,4,5,6,16,32")
    ap.add_argument("--fmt", default=None, help="override the workload's format (int4, int8, nvfp4)")
    args = ap.parse_args(argv)
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from synth import make_workload
    wl = make_workload(args.workload, rows=args.rows)
    dev = torch.device("cuda:0")
    tdt = torch.bfloat16 if wl.x_dtype == "bf16" else torch.float32
    x = torch.from_numpy(wl.x).to(dev).to(tdt)
    W = torch.from_numpy(wl.W).to(dev).to(torch.bfloat16 if wl.w_dtype == "bf16" else torch.float32)
    scale = torch.from_numpy(wl.scale).to(dev)
    fmt = args.fmt or (wl.fmt if wl.fmt == "nvfp4" else f"int{wl.bits}")
    res = ablation(x, W, scale, [int(r) for r in args.ranks.split(",")], fmt=fmt)
    res["workload"] = args.workload
    print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
