"""Benchmark of the SVDQuant inference linear on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the operator's hot path over one batch: the fused
activation pass (smoothing, per-tensor max, codes, down-projection) and the
residual tensor-core GEMM with the low-rank + bias epilogue, both through the
C ABI. The weight split (svdq_prepare) is timed once, separately. Inputs are
synthetic and seeded (synth/), resident in HBM when the timed region starts.
The run keeps R buffer sets (x, prepared weight, codes, down, Y) spanning at
least three L2 sizes and step i uses set i % R, so no step finds its inputs in
L2; the K steps run back to back (one CUDA graph per step when capture works)
between one pair of CUDA events.

value     whole-job TOPS (2BMN residual ops + 2Br(M+N) low-rank flops per step)
e2e       the same metric through svdq_linear with pinned host x copied in and
          Y copied out inside the timed region
roofline  the GEMM kernel against the dense int8 tensor peak (measured bf16
          GEMM peak x 2, the nominal int8:bf16 ratio)
cpu_baseline / --impl reference   the float64 CPU oracle, timed on host cores

Multi-GPU: replicas only (the operator is single-GPU); each rank runs the same
workload on its own device, the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "svdq_linear TOPS and GB/s at 1 B200; % of roofline (HBM or int8/FP4 peak)"
DEFAULT_WORKLOAD = "dit_attn_4096x3072x3072_int4"
L2_ROTATE_BYTES = 3 * (126 << 20)   # the buffer sets of a run span three L2 sizes at least
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- helpers
def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def workload_ops(B, M, N, rank):
    return 2.0 * B * M * N + 2.0 * B * rank * (M + N)


def alg_bytes(B, M, N, rank, fmt, bits, bias):
    """Algorithmic bytes of one step: bf16 x, weight codes (+scales), bf16 factors,
    fp32 scale, bias, bf16 Y."""
    if fmt in ("nvfp4", "mxfp4"):
        wbytes = M * N * (0.5 + (1.0 / 16.0 if fmt == "nvfp4" else 1.0 / 32.0))
    else:
        wbytes = M * N * (0.5 if bits <= 4 else 1.0)
    return (B * M * 2 + wbytes + 2 * rank * (M + N) + 4 * M + (2 * N if bias else 0)
            + B * N * 2)


def gemm_alg_bytes(B, M, N, rank, fmt, bits, bias):
    """Algorithmic bytes of one GEMM launch: weight codes (+ scales), the bf16 up
    factor, the activation codes (+ scales) and the bf16 down tile it reads, bias,
    and the bf16 Y it writes."""
    if fmt in ("nvfp4", "mxfp4"):
        per = 0.5 + (1.0 / 16.0 if fmt == "nvfp4" else 1.0 / 32.0)
        wbytes, abytes = M * N * per, B * M * per
    else:
        wbytes, abytes = M * N * (0.5 if bits <= 4 else 1.0), B * M
    return wbytes + 2 * rank * N + abytes + 2 * B * rank + (2 * N if bias else 0) + 2 * B * N


def gemm_alg_ops(B, M, N, rank):
    return 2.0 * B * M * N + 2.0 * B * rank * N


def read_profile_traffic(workload, sources):
    """DRAM traffic per launch of the GEMM kernel from the committed ncu summary of
    this workload, if it was taken on these very kernel sources (a sha256 of the
    sources is recorded beside it), else None."""
    import hashlib
    try:
        text = open(os.path.join(ROOT, "profiles", f"gemm_pair_{workload}.md")).read()
    except OSError:
        return None
    h = hashlib.sha256()
    for src in sources:
        h.update(open(src, "rb").read())
    vals = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            vals[k.strip()] = v.strip().split()[0].strip("`") if v.strip() else ""
    if vals.get("kernel_source_sha256") != h.hexdigest():
        return None
    try:
        return float(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []
        self.t = None
        self.clocks = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1])); smax.append(float(parts[2])); power.append(float(parts[3]))
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


def cpu_oracle_rate(wl, budget_s=12.0, rows=None):
    """Time the float64 oracle (prepared-operand linear, in the workload's own
    format) on the host cores over a bounded sample; returns (TOPS, seconds,
    cores, sample description)."""
    import numpy as np
    from oracle import codes as ocodes
    from oracle import prepared as oprep

    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count() or 1
    rng = np.random.default_rng(0)
    B, M, N, r = wl.B, wl.M, wl.N, wl.rank
    rows = rows or min(B, 512)
    ld = (rng.standard_normal((M, r)) * 0.01).astype(np.float64)
    L2 = (rng.standard_normal((r, N)) * 0.01).astype(np.float64)
    x = wl.x[:rows]
    if wl.fmt == "int":
        cw = rng.integers(-7, 8, (N, M)).astype(np.int8)

        def once():
            q, s_x, _ = ocodes.act_codes_int_fp32(x, wl.scale, wl.bits)
            oprep.linear_int(x, ld, L2, q, s_x, cw, 0.01)
        what = "fp32-mode codes + float64 integer product + low-rank"
    elif wl.fmt == "nvfp4":
        from oracle import nvfp4 as onv
        cw = rng.integers(0, 16, (N, M)).astype(np.uint8)
        sfw = rng.integers(0x20, 0x48, (N, M // 16)).astype(np.uint8)

        def once():
            ca, sa, gx = onv.quantize(ocodes.smooth_fp32(x, wl.scale))
            oprep.linear_nvfp4(x, ld, L2, ca, sa, gx, cw, sfw, 448.0)
        what = "NVFP4 block quantisation + float64 block-scaled product + low-rank"
    else:
        from oracle import mxfp4 as omx
        cw = rng.integers(0, 16, (N, M)).astype(np.uint8)
        sfw = rng.integers(121, 127, (N, M // 32)).astype(np.uint8)

        def once():
            ca, sa = omx.quantize(ocodes.smooth_fp32(x, wl.scale))
            oprep.linear_mxfp4(x, ld, L2, ca, sa, cw, sfw)
        what = "MXFP4 block quantisation + float64 block-scaled product + low-rank"
    t0 = time.perf_counter()
    ops = 0.0
    reps = 0
    while True:
        once()
        ops += workload_ops(rows, M, N, r)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    sample = (f"{reps} pass(es) of the oracle's prepared-operand linear ({what}) over {rows} of {B} rows "
              f"of {wl.name}")
    return ops / dt / 1e12, dt, cores, sample


# ------------------------------------------------------------- reference
def run_reference(args, wl_name):
    """Reference arm: the CPU oracle, timed on the host cores, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from synth import make_workload
    wl = make_workload(wl_name)
    per_step = max(0.5, 60.0 / max(args.steps + args.warmup, 1))
    for _ in range(args.warmup):
        cpu_oracle_rate(wl, budget_s=0.0, rows=64)
    vals, secs = [], 0.0
    cores, sample = 1, ""
    for _ in range(args.steps):
        v, dt, cores, sample = cpu_oracle_rate(wl, budget_s=per_step, rows=256)
        vals.append(v)
        secs += dt
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * secs / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl_name, "B": wl.B, "M": wl.M, "N": wl.N, "rank": wl.rank,
                   "fmt": f"{wl.fmt}{wl.bits}" if wl.fmt == "int" else wl.fmt},
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sets", type=int, default=0,
                    help="rotating buffer sets (default: enough to span three L2 sizes)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args, args.workload)

    import numpy as np
    import torch
    import torch.distributed as dist

    import rank_bit_residual_b200 as rb
    from synth import make_workload

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    wl = make_workload(args.workload)
    B, M, N, r = wl.B, wl.M, wl.N, wl.rank
    fmt = f"int{wl.bits}" if wl.fmt == "int" else wl.fmt
    xdt = torch.bfloat16 if wl.x_dtype == "bf16" else torch.float32
    x = torch.from_numpy(wl.x).to(xdt).to(dev)
    W = torch.from_numpy(wl.W).to(xdt).to(dev)
    scale = torch.from_numpy(wl.scale).to(dev)
    bias = torch.from_numpy(wl.bias).to(torch.bfloat16).to(dev) if wl.bias is not None else None

    # one-time split (timed separately)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    w = rb.svdq_prepare(W, scale, r, fmt, seed=0)
    torch.cuda.synchronize()
    prepare_ms = 1000.0 * (time.perf_counter() - t0)
    wgs_of = (lambda wt: wt.w_scale) if wl.fmt == "nvfp4" else (lambda wt: None)

    # R buffer sets (x, weight, codes, down, Y) whose union is several times
    # the L2 size: step i runs on set i % R, so no step finds its inputs in L2
    bytes_set = alg_bytes(B, M, N, r, wl.fmt, wl.bits, wl.bias is not None) + B * M  # + act codes
    R = int(min(64, max(2, -(-L2_ROTATE_BYTES // bytes_set)))) if args.sets <= 0 else args.sets
    sets = []
    for k in range(R):
        wk = w if k == 0 else rb.svdq_prepare(W, scale, r, fmt, seed=0)
        xk = x if k == 0 else x.clone()
        c, sfk, asc, dn = rb.svdq_quantize_act(xk, scale, fmt, ld=wk.ld if r else None,
                                               w_global_scale=wgs_of(wk))
        yk = torch.empty((B, N), dtype=torch.bfloat16, device=dev)
        sets.append((wk, xk, c, sfk, asc, dn, yk, rb.LinearWorkspace()))
    del W
    y = sets[0][6]
    stream = torch.cuda.current_stream()

    def act_stage(k):
        wk, xk, c, sfk, asc, dn, yk, _ = sets[k]
        rb.svdq_quantize_act_into(xk, scale, fmt, wk.ld if r else None, c, sfk, asc, dn,
                                  w_global_scale=wgs_of(wk))

    def gemm_stage(k):
        wk, xk, c, sfk, asc, dn, yk, _ = sets[k]
        rb.svdq_residual_linear(wk, c, sfk, asc, dn, bias=bias, out=yk)

    def step(k, rows=None):
        # the operator through its C-ABI call: activation pass, then the GEMM
        # (for B <= 128 a dependent launch whose weight loads overlap the first)
        wk, xk, c, sfk, asc, dn, yk, wsk = sets[k]
        if rows is None:
            rb.svdq_linear(wk, xk, bias=bias, out=yk, workspace=wsk)
        else:
            rb.svdq_linear(wk, xk[:rows], bias=bias, out=yk[:rows], workspace=wsk)

    for i in range(max(args.warmup, R)):
        step(i % R)
    torch.cuda.synchronize()
    assert rb.svdq_check_status() == rb.SVDQ_OK

    # one CUDA graph per buffer set holds a whole step (the activation pass and
    # the GEMM with their launches); plain stream launches if capture fails
    def capture_seq(fn, n):
        """One CUDA graph holding n consecutive calls fn(i), i = 0 .. n-1 (set i % R)."""
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                for i in range(n):
                    fn(i)
        stream.wait_stream(cap)
        g.replay()
        torch.cuda.synchronize()
        assert rb.svdq_check_status() == rb.SVDQ_OK
        return g

    graph_mode = {"ok": True}

    def time_calls(fn, K, sampler=None):
        """Device time (ms) of K calls fn(i) back to back, set i % R. The calls are
        captured in CUDA graphs of L calls (L a multiple of R), replayed between one
        pair of CUDA events, so the host's launch cost is not inside the interval."""
        L = R * max(1, 64 // R)
        graphs_ = None
        if graph_mode["ok"]:
            try:
                graphs_ = (capture_seq(fn, min(L, K)), capture_seq(fn, K % L) if K > L and K % L else None)
            except Exception as e:  # noqa: BLE001 - any capture failure falls back to launches
                print(f"bench: CUDA graph capture unavailable ({type(e).__name__}: {e}); stream launches",
                      file=sys.stderr)
                graph_mode["ok"] = False
                torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        if sampler is not None:
            sampler.start()
            time.sleep(0.2)
        e0.record(stream)
        if graphs_ is not None:
            for _ in range(K // L if K >= L else 1):
                graphs_[0].replay()
            if graphs_[1] is not None:
                graphs_[1].replay()
        else:
            for i in range(K):
                fn(i % R)
        e1.record(stream)
        torch.cuda.synchronize()
        if sampler is not None:
            sampler.clocks = sampler.stop()
        if world > 1:
            dist.barrier()
        return e0.elapsed_time(e1)

    K = args.steps
    sampler = ClockSampler(local)
    total_ms = time_calls(lambda i: step(i % R), K, sampler)
    clocks = sampler.clocks
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    ops_step = workload_ops(B, M, N, r)
    value = world * K * ops_step / (total_ms * 1e-3) / 1e12
    ms_per_step = total_ms / K

    # decode shapes: the shorter batches of the sweep (the first rows of the same
    # x, same weights and rotation), each timed the same way
    sweep = None
    if args.workload.startswith("decode_") and B == 128:
        sweep = []
        peaks0, _ = load_peaks()
        for rows in (1, 16):
            for i in range(max(args.warmup, R)):
                step(i % R, rows)
            torch.cuda.synchronize()
            us = time_calls(lambda i, rows=rows: step(i % R, rows), K) / K * 1e3
            byt = alg_bytes(rows, M, N, r, wl.fmt, wl.bits, wl.bias is not None)
            t_mem = byt / (peaks0["hbm_gbs"] * 1e9)
            sweep.append({"B": rows, "us_per_step": us, "gbs": byt / (us * 1e-6) / 1e9,
                          "tops": workload_ops(rows, M, N, r) / (us * 1e-6) / 1e12,
                          "hbm_roofline_frac": t_mem / (us * 1e-6), "alg_bytes": byt})
        assert rb.svdq_check_status() == rb.SVDQ_OK

    # consecutive linears (square shapes): layer k of a chain of R runs on set k's
    # weights and reads layer k-1's Y, so the weights stream from HBM while the
    # activations stay in L2, as in a network; timed plain and with each layer's
    # activation pass a programmatic dependent of the previous layer's GEMM
    chain = None
    if M == N:
        def chain_graph(pdl, rows):
            def run():
                prev = x[:rows]
                for k in range(R):
                    wk, _, _, _, _, _, yk, wsk = sets[k]
                    rb.svdq_linear(wk, prev, bias=bias, out=yk[:rows], workspace=wsk, pdl=pdl and k > 0)
                    prev = yk[:rows]
            run()
            torch.cuda.synchronize()
            cap = torch.cuda.Stream()
            cap.wait_stream(stream)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                run()
            stream.wait_stream(cap)
            return g

        def time_chain(pdl, rows, reps):
            g = chain_graph(pdl, rows)
            g.replay()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) * 1e3 / (reps * R)

        chain = {"layers_per_chain": R, "note": "us per linear, chains of R layers of this shape "
                                               "captured in one CUDA graph; layer 0 plain in both"}
        for rows in ((1, B) if args.workload.startswith("decode_") else (B,)):
            reps = max(3, min(50, (200 * 1000) // max(1, R * int(ms_per_step * 1e3 + 1))))
            plain = time_chain(False, rows, reps)
            pdl = time_chain(True, rows, reps)
            chain[f"B={rows}"] = {"plain_us": plain, "pdl_us": pdl, "saved_us": plain - pdl}
        assert rb.svdq_check_status() == rb.SVDQ_OK

    # each stage alone, Ks launches back to back on the rotating sets: the GEMM's
    # average launch duration is the roofline line's
    Kg = max(20, min(K, 400))
    gemm_avg_ms = time_calls(lambda i: gemm_stage(i % R), Kg) / Kg
    act_avg_ms = time_calls(lambda i: act_stage(i % R), Kg) / Kg
    # the step the parity check reads: set 0 once more
    step(0)
    torch.cuda.synchronize()

    # parity on sampled rows of the timed output (oracle from the prepared buffers)
    parity = None
    if rank == 0:
        from oracle import codes as ocodes
        from oracle import prepared as oprep
        rows = np.random.default_rng(1).choice(B, size=min(B, 48), replace=False)
        ld = w.ld.float().cpu().numpy()[: w.rank_pad].T
        L2 = w.lu.float().cpu().numpy()[:, : w.rank_pad].T
        if wl.fmt == "int":
            q, s_x, _ = ocodes.act_codes_int_fp32(wl.x, wl.scale, wl.bits)
            cw = w.codes.view(torch.int8).cpu().numpy().reshape(N, M)
            want = oprep.linear_int(wl.x[rows], ld, L2, q[rows], s_x, cw, float(w.w_scale[0].item()),
                                    wl.bias)
        elif wl.fmt == "mxfp4":
            from oracle import mxfp4 as omx
            from oracle import nvfp4 as onv
            ca, sa = omx.quantize(ocodes.smooth_fp32(wl.x[rows], wl.scale))
            cw = onv.unpack_nibbles(w.codes.cpu().numpy().reshape(N, M // 2))
            sfw = onv.sf_unswizzle(w.sf.cpu().numpy(), N, M // 32)
            want = oprep.linear_mxfp4(wl.x[rows], ld, L2, ca, sa, cw, sfw, wl.bias)
        else:
            from oracle import nvfp4 as onv
            xs = ocodes.smooth_fp32(wl.x, wl.scale)
            ca, sa, gx = onv.quantize(xs)
            cw = onv.unpack_nibbles(w.codes.cpu().numpy().reshape(N, M // 2))
            sfw = onv.sf_unswizzle(w.sf.cpu().numpy(), N, M // 16)
            want = oprep.linear_nvfp4(wl.x[rows], ld, L2, ca[rows], sa[rows], gx, cw, sfw,
                                      float(w.w_scale[0].item()), wl.bias)
        got = y[torch.from_numpy(rows).to(dev)].float().cpu().numpy()
        rel = float(np.linalg.norm(got - want) / np.linalg.norm(want))
        parity = {"rows_sampled": int(len(rows)), "rel_fro": rel, "y": "bf16 (rounding included)",
                  "max_rel": float(np.max(np.abs(got - want)) / np.max(np.abs(want)))}

    # end to end through svdq_linear with host buffers
    x_host = x.cpu().pin_memory()
    y_host = torch.empty((B, N), dtype=torch.bfloat16).pin_memory()
    xd = torch.empty_like(x)
    ws = rb.LinearWorkspace()
    Ke = max(3, min(50, K))
    for _ in range(3):
        xd.copy_(x_host, non_blocking=True)
        rb.svdq_linear(w, xd, bias=bias, out=y, workspace=ws)
        y_host.copy_(y, non_blocking=True)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(Ke):
        xd.copy_(x_host, non_blocking=True)
        rb.svdq_linear(w, xd, bias=bias, out=y, workspace=ws)
        y_host.copy_(y, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(e2e_ms, op=dist.ReduceOp.MAX)
    e2e_value = world * Ke * ops_step / (float(e2e_ms.item()) * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    # a contraction takes the peak of its own dtype: measured bf16 x nominal ratio
    ratio = 4.0 if wl.fmt != "int" else 2.0
    lowp_peak = ratio * peaks["bf16_tflops"]
    g_ops = gemm_alg_ops(B, M, N, r)
    achieved = g_ops / (gemm_avg_ms * 1e-3) / 1e12
    csrc = os.path.join(ROOT, "rank_bit_residual_b200", "csrc")
    traffic = read_profile_traffic(args.workload, [os.path.join(csrc, f) for f in
                                                   ("gemm_pair.cu", "gemm_common.cuh", "ptx.cuh")]) \
        if B > 128 else None
    bytes_step = alg_bytes(B, M, N, r, wl.fmt, wl.bits, wl.bias is not None)
    if B <= 128:
        # short batch: the GEMM streams the weights; its roofline is HBM
        gb = gemm_alg_bytes(B, M, N, r, wl.fmt, wl.bits, wl.bias is not None)
        roof = {"bound": "hbm",
                "kernel": "skinny_kernel<" + (wl.fmt.upper() if wl.fmt != "int" else
                                              ("INT4 packed" if wl.bits <= 4 else "INT8")) +
                          "> (split-K clusters, residual + bf16 up-projection)",
                "duration_us": gemm_avg_ms * 1e3,
                "timing": "Kg launches back to back on rotating sets (CUDA graphs) between one CUDA event pair",
                "achieved": gb / (gemm_avg_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gb / (gemm_avg_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "traffic": None,
                "alg_bytes_per_launch": gb,
                "peak_source": f"{peak_src} HBM copy bandwidth"}
    else:
        roof = {"bound": "tensor",
                "kernel": "gemm_pair_kernel" + (f"<{wl.fmt.upper()}> (e2m1 block-scaled residual + bf16 "
                                                "up-projection)" if wl.fmt != "int" else
                                                "<INT> (int8 residual + bf16 up-projection)"),
                "duration_us": gemm_avg_ms * 1e3,
                "timing": "Kg launches back to back on rotating sets (CUDA graphs) between one CUDA event pair",
                "achieved": achieved, "peak": lowp_peak, "unit": "TFLOP/s",
                "frac": achieved / lowp_peak, "traffic": traffic,
                "peak_source": (f"{peak_src} bf16 GEMM burst x {ratio:g} "
                                f"(nominal {'fp4' if ratio == 4 else 'int8'}:bf16)")}
    t_rf = max(bytes_step / (peaks["hbm_gbs"] * 1e9),
               (2.0 * B * M * N) / (lowp_peak * 1e12) + (2.0 * B * r * (M + N)) / (peaks["bf16_tflops"] * 1e12))

    out = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e2m1" if wl.fmt != "int" else "int8",
        "data": "synthetic",
        "config": {"workload": args.workload, "B": B, "M": M, "N": N, "rank": r, "fmt": fmt,
                   "x": wl.x_dtype, "y": "bf16", "bias": wl.bias is not None,
                   "l2": f"inputs larger than L2: {R} rotating buffer sets of {bytes_set / 1e6:.0f} MB",
                   "launch": ("CUDA graphs of many steps" if graph_mode["ok"] else "stream launches"),
                   "parallelism": f"replicas{world}"},
        "gbs": bytes_step / (ms_per_step * 1e-3) / 1e9,
        "step_roofline": {"t_roofline_us": t_rf * 1e6, "frac": t_rf / (ms_per_step * 1e-3),
                          "alg_bytes": bytes_step, "ops": ops_step},
        "stages_ms": {"act": act_avg_ms, "gemm": gemm_avg_ms,
                      "note": "each stage alone, launched back to back on the rotating sets (CUDA "
                              "graphs of many launches between one event pair); in a step the GEMM "
                              "of a short batch overlaps the activation pass (dependent launch)"},
        "roofline": roof,
        "prepare_ms": prepare_ms,
        "parity": parity,
        "e2e": {"value": e2e_value, "unit": "TOPS", "h2d_bytes_per_step": int(x.numel() * x.element_size()),
                "d2h_bytes_per_step": int(y.numel() * y.element_size()), "steps": Ke,
                "call": "svdq_linear (pinned host x -> device, Y -> pinned host)"},
        "gpu_launches": 3 * K,   # per step: activation stats, activation codes, residual GEMM
        "sweep": sweep,
        "chain": chain,
        "clocks": clocks,
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        v, dt, cores, sample = cpu_oracle_rate(wl)
        out["cpu_baseline"] = {"value": v, "unit": "TOPS", "cores": cores, "kind": "oracle",
                               "sample": sample, "seconds": dt}
    elif rank == 0:
        out["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
