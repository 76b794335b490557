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

The smoothing scale's migration strength (the "SVDQuant parameter configuration
guide", step 3 "choose and tune the parameters": iter_smooth.alpha) is chosen the
same way: select_alpha computes the scale of each candidate strength on the GPU
(svdq_smooth_scale) from calibration activations, runs the two-branch linear at the
given rank, and keeps the strength with the smallest output error.

The diagonal fold of "Contraction-Gauge Preconditioning for Quantized Matrix
Multiplication" (svdq_fold_scale: the geometric program's optimal shared fold of
x @ W under per-tensor grids) is a scale of its own; fold_vs_alpha runs the
two-branch linear with it beside the migration strengths.

    python -m rank_bit_residual_b200.ablation [--workload NAME] [--rows B] [--ranks 0,1,2,...]
                                              [--alphas 0.25,0.5,0.75,0.9] [--fold]

prints one JSON object (errors per variant and rank, singular values, timings, the
error per migration strength, and with --fold the fold's errors).
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

from . import svdq_fold_scale, svdq_linear, svdq_prepare, svdq_smooth_scale


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


def select_alpha(x_calib: torch.Tensor, W: torch.Tensor, rank: int, fmt: str = "int4",
                 alphas: Sequence[float] = (0.25, 0.5, 0.75, 0.9), x_eval: Optional[torch.Tensor] = None,
                 seed: int = 0) -> Dict:
    """The migration strength with the smallest two-branch output error.

    The scale of each strength comes from the calibration activations x_calib; the
    error is measured on x_eval (default: x_calib). Returns the error per strength,
    the chosen strength and its scale.
    """
    xe = x_calib if x_eval is None else x_eval
    ref = xe.double() @ W.double()
    table = {}
    best = None
    for a in alphas:
        scale = svdq_smooth_scale(x_calib, W, float(a))
        w = svdq_prepare(W, scale, rank, fmt, seed=seed)
        err = rel_fro(svdq_linear(w, xe, out_dtype=torch.float32), ref)
        table[float(a)] = err
        if best is None or err < best[1]:
            best = (float(a), err, scale)
    return {"errors": table, "alpha": best[0], "error": best[1], "scale": best[2]}


def fold_vs_alpha(x_calib: torch.Tensor, W: torch.Tensor, ranks: Sequence[int], fmt: str = "int4",
                  alphas: Sequence[float] = (0.25, 0.5, 0.75, 0.9), bits: int = 4,
                  x_eval: Optional[torch.Tensor] = None, seed: int = 0) -> Dict:
    """Two-branch output errors with the geometric program's fold (svdq_fold_scale of
    the calibration activations, per-tensor grids of `bits`) and with each migration
    strength, at each rank; error on x_eval (default x_calib)."""
    xe = x_calib if x_eval is None else x_eval
    ref = xe.double() @ W.double()
    scales = {"fold": svdq_fold_scale(x_calib, W, bits)}
    for a in alphas:
        scales[f"alpha={float(a):g}"] = svdq_smooth_scale(x_calib, W, float(a))
    out = {}
    for name, sc in scales.items():
        out[name] = {int(r): rel_fro(svdq_linear(svdq_prepare(W, sc, int(r), fmt, seed=seed), xe,
                                                 out_dtype=torch.float32), ref) for r in ranks}
    return out


def main(argv: Optional[Sequence[str]] = None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="dit_attn_4096x3072x3072_int4")
    ap.add_argument("--rows", type=int, default=None, help="keep only the first rows of x")
    ap.add_argument("--ranks", default="0,1,2,3,4,5,6,16,32")
    ap.add_argument("--fmt", default=None, help="override the workload's format (int4, int8, nvfp4, mxfp4)")
    ap.add_argument("--alphas", default="0.25,0.5,0.75,0.9",
                    help="migration strengths to compare at the largest rank (empty: skip)")
    ap.add_argument("--fold", action="store_true",
                    help="also run the geometric program's fold beside the migration strengths")
    args = ap.parse_args(argv)
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from synth import make_workload
    wl = make_workload(args.workload, rows=args.rows)
    dev = torch.device("cuda:0")
    tdt = torch.bfloat16 if wl.x_dtype == "bf16" else torch.float32
    x = torch.from_numpy(wl.x).to(dev).to(tdt)
    W = torch.from_numpy(wl.W).to(dev).to(torch.bfloat16 if wl.w_dtype == "bf16" else torch.float32)
    scale = torch.from_numpy(wl.scale).to(dev)
    fmt = args.fmt or (wl.fmt if wl.fmt != "int" else f"int{wl.bits}")
    ranks = [int(r) for r in args.ranks.split(",")]
    res = ablation(x, W, scale, ranks, fmt=fmt)
    res["workload"] = args.workload
    if args.alphas:
        sel = select_alpha(x, W, max(ranks), fmt, [float(a) for a in args.alphas.split(",")])
        res["alpha_selection"] = {"rank": max(ranks), "errors": sel["errors"], "alpha": sel["alpha"]}
    if args.fold:
        alphas = [float(a) for a in args.alphas.split(",")] if args.alphas else []
        bits = int(fmt[3:]) if fmt.startswith("int") else 4
        res["fold_vs_alpha"] = fold_vs_alpha(x, W, sorted({0, max(ranks)}), fmt, alphas, bits)
    print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
