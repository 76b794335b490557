"""Benchmark of the SVDQuant inference linear on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--configs all|none] [--impl reference]

A step is one pass of the operator's hot path over one batch: the fused
activation pass (smoothing, per-tensor max, codes, down-projection) and the
residual tensor-core GEMM with the low-rank + bias epilogue, both through the
C ABI. The weight split (svdq_prepare) is timed separately. Inputs are
synthetic and seeded (synth/), resident in HBM when the timed region starts.
The run keeps R buffer sets (x, prepared weight, codes, down, Y) spanning at
least three L2 sizes and step i uses set i % R, so no step finds its inputs in
L2; the K steps run back to back (CUDA graphs of many steps) between one pair
of CUDA events. Clocks are sampled over a window of back-to-back steps that
contains the timed region (a few hundred ms of steps run just before it on the
same stream, with no gap), so the sampler sees the GPU under that load.

The headline workload is the largest single-GPU configuration, x[8192, 12288]
with W[12288, 3072], INT4, rank 32. With --configs all (the default for the
default workload) the same line carries one record per other configuration
of the sweep under "configs": the tiny case, the DiT attention and MLP
projections, the decode sweep B in {1, 16, 128} in INT4 / NVFP4 / MXFP4 and the
large shape in INT4 / INT8 / NVFP4 / MXFP4 at ranks 32 and 128, each with its
time per step, TOPS, GB/s, step and kernel roofline fractions and the time of
svdq_prepare for its weight.

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
DEFAULT_WORKLOAD = "large_8192x12288x3072_int4_r32"
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
            q, s_x, _ = ocodes.act_codes_int(x, wl.scale, wl.bits)
            oprep.linear_int(x, ld, L2, q, s_x, cw, 0.01)
        what = "exactly rounded INT codes + float64 integer product + low-rank"
    elif wl.fmt == "nvfp4":
        from oracle import nvfp4 as onv
        cw = rng.integers(0, 16, (N, M)).astype(np.uint8)
        sfw = rng.integers(0x20, 0x48, (N, M // 16)).astype(np.uint8)

        def once():
            ca, sa, gx = onv.quantize(x, div=wl.scale)
            oprep.linear_nvfp4(x, ld, L2, ca, sa, gx, cw, sfw, 448.0)
        what = "NVFP4 block quantisation + float64 block-scaled product + low-rank"
    else:
        from oracle import mxfp4 as omx
        cw = rng.integers(0, 16, (N, M)).astype(np.uint8)
        sfw = rng.integers(121, 127, (N, M // 32)).astype(np.uint8)

        def once():
            ca, sa = omx.quantize(x, div=wl.scale)
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


# ------------------------------------------------------------- configs
# Per-configuration records of the default run, in the order they are measured
# (the large-shape variants first: they share the headline's draw of x and W).
EXTRA_CONFIGS = [
    ("large_8192x12288x3072_int4_r128", None),
    ("large_8192x12288x3072_int8_r32", None),
    ("large_8192x12288x3072_int8_r128", None),
    ("large_8192x12288x3072_nvfp4_r32", None),
    ("large_8192x12288x3072_nvfp4_r128", None),
    ("large_8192x12288x3072_mxfp4_r32", None),
    ("large_8192x12288x3072_mxfp4_r128", None),
    ("dit_attn_4096x3072x3072_int4", None),
    ("dit_mlp_4096x3072x12288_nvfp4", None),
    ("dit_mlp_4096x3072x12288_mxfp4", None),
    ("decode_128x4096x4096_int4", 128),
    ("decode_128x4096x4096_int4", 16),
    ("decode_128x4096x4096_int4", 1),
    ("decode_128x4096x4096_nvfp4", 128),
    ("decode_128x4096x4096_nvfp4", 16),
    ("decode_128x4096x4096_nvfp4", 1),
    ("decode_128x4096x4096_mxfp4", 128),
    ("decode_128x4096x4096_mxfp4", 16),
    ("decode_128x4096x4096_mxfp4", 1),
    ("tiny_16x256x128_int4", None),
]
EXTRA_TIMED_MS = 150.0   # device time each extra record's timed region aims for
SOAK_MS = 400.0          # back-to-back steps just before a sampled timed region


def launches_per_step(wl) -> int:
    """Kernels one svdq_linear call launches: one for up to 16 rows with INT weights
    (the single-launch decode kernel, whose shared memory holds every decode shape
    benched here), else two for the activation pass and one GEMM."""
    return 1 if (wl.fmt == "int" and wl.B <= 16) else 3


def fmt_name(wl):
    return f"int{wl.bits}" if wl.fmt == "int" else wl.fmt


def config_of(wl, name, extra=None):
    """The line's config dict (the same keys in both arms)."""
    c = {"workload": name, "B": wl.B, "M": wl.M, "N": wl.N, "rank": wl.rank, "fmt": fmt_name(wl),
         "x": wl.x_dtype, "y": "bf16", "bias": wl.bias is not None}
    c.update(extra or {})
    return c


# ------------------------------------------------------------- reference
def run_reference(args, wl_name):
    """Reference arm: the CPU oracle, timed on the host cores, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from synth import make_workload
    wl = make_workload(wl_name, rows=args.rows)
    per_step = max(0.5, 60.0 / max(args.steps + args.warmup, 1))
    for _ in range(args.warmup):
        cpu_oracle_rate(wl, budget_s=0.0, rows=16)
    vals, secs = [], 0.0
    cores, sample = 1, ""
    for _ in range(args.steps):
        v, dt, cores, sample = cpu_oracle_rate(wl, budget_s=per_step, rows=128)
        vals.append(v)
        secs += dt
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * secs / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, wl_name, {
            "l2": "host memory (CPU oracle)", "launch": "host, bounded row sample per step",
            "parallelism": f"replicas{args.gpus}"}),
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ engine
class Engine:
    """One device, one stream; rotating buffer sets per workload; CUDA-graph timing."""

    def __init__(self, dev, world, rank, local):
        import torch
        self.torch = torch
        self.dev, self.world, self.rank, self.local = dev, world, rank, local
        self.stream = torch.cuda.current_stream()
        self.graph_ok = True
        self._prep_cache = None   # (workload name, prepared weights of the sets, prepare_ms)

    # -- setup ---------------------------------------------------------------
    def setup(self, name, rows=None, nsets=0):
        """Buffer sets for a workload: weights prepared on the device, x, codes, down, Y."""
        import torch
        import rank_bit_residual_b200 as rb
        from synth import make_workload
        wl = make_workload(name)
        if rows is not None:
            wl = wl.rows(rows)
        B, M, N, r = wl.B, wl.M, wl.N, wl.rank
        fmt = fmt_name(wl)
        xdt = torch.bfloat16 if wl.x_dtype == "bf16" else torch.float32
        x = torch.from_numpy(wl.x).to(xdt).to(self.dev)
        scale = torch.from_numpy(wl.scale).to(self.dev)
        bias = torch.from_numpy(wl.bias).to(torch.bfloat16).to(self.dev) if wl.bias is not None else None
        bytes_set = alg_bytes(B, M, N, r, wl.fmt, wl.bits, wl.bias is not None) + B * M   # + act codes
        R = int(min(64, max(2, -(-L2_ROTATE_BYTES // bytes_set)))) if nsets <= 0 else nsets
        if self._prep_cache is not None and self._prep_cache[0] == name and len(self._prep_cache[1]) >= R:
            weights, prepare_ms = self._prep_cache[1][:R], self._prep_cache[2]
        else:
            self._prep_cache = None
            W = torch.from_numpy(wl.W).to(xdt).to(self.dev)
            weights, times = [], []
            for k in range(R):
                torch.cuda.synchronize()
                t0 = time.perf_counter()
                weights.append(rb.svdq_prepare(W, scale, r, fmt, seed=0))
                torch.cuda.synchronize()
                times.append(1000.0 * (time.perf_counter() - t0))
            del W
            # the first call of a process also pays one-time set-up; report the later ones
            prepare_ms = statistics.median(times[1:]) if len(times) > 1 else times[0]
            self._prep_cache = (name, weights, prepare_ms)
        wgs = (lambda wt: wt.w_scale) if wl.fmt == "nvfp4" else (lambda wt: None)
        sets = []
        for k in range(R):
            wk = weights[k]
            xk = x if k == 0 else x.clone()
            c, sfk, asc, dn = rb.svdq_quantize_act(xk, scale, fmt, ld=wk.ld if r else None,
                                                   w_global_scale=wgs(wk))
            yk = torch.empty((B, N), dtype=torch.bfloat16, device=self.dev)
            sets.append((wk, xk, c, sfk, asc, dn, yk, rb.LinearWorkspace()))
        return {"wl": wl, "name": name, "fmt": fmt, "x": x, "scale": scale, "bias": bias, "R": R,
                "sets": sets, "bytes_set": bytes_set, "prepare_ms": prepare_ms, "wgs": wgs}

    # -- calls -----------------------------------------------------------------
    @staticmethod
    def step(ctx, k):
        import rank_bit_residual_b200 as rb
        wk, xk, c, sfk, asc, dn, yk, wsk = ctx["sets"][k % ctx["R"]]
        rb.svdq_linear(wk, xk, bias=ctx["bias"], out=yk, workspace=wsk)

    @staticmethod
    def act_stage(ctx, k):
        import rank_bit_residual_b200 as rb
        wk, xk, c, sfk, asc, dn, yk, _ = ctx["sets"][k % ctx["R"]]
        rb.svdq_quantize_act_into(xk, ctx["scale"], ctx["fmt"], wk.ld if ctx["wl"].rank else None, c, sfk, asc,
                                  dn, w_global_scale=ctx["wgs"](wk))

    @staticmethod
    def gemm_stage(ctx, k):
        import rank_bit_residual_b200 as rb
        wk, xk, c, sfk, asc, dn, yk, _ = ctx["sets"][k % ctx["R"]]
        rb.svdq_residual_linear(wk, c, sfk, asc, dn, bias=ctx["bias"], out=yk)

    # -- timing ----------------------------------------------------------------
    def _capture(self, fn, n):
        torch = self.torch
        import rank_bit_residual_b200 as rb
        cap = torch.cuda.Stream()
        cap.wait_stream(self.stream)
        with torch.cuda.stream(cap):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                for i in range(n):
                    fn(i)
        self.stream.wait_stream(cap)
        g.replay()
        torch.cuda.synchronize()
        assert rb.svdq_check_status() == rb.SVDQ_OK
        return g

    def time_calls(self, fn, K, R, sampler=None, soak_ms=0.0, est_ms=None):
        """Device time (ms) of K calls fn(i) back to back, captured in CUDA graphs of
        L calls (L a multiple of R) and replayed between one pair of CUDA events. With
        a sampler, soak_ms of the same calls run first on the stream with no gap, and
        the sampler covers soak and timed region."""
        torch = self.torch
        L = R * max(1, 64 // R)
        gs = None
        if self.graph_ok:
            try:
                gs = (self._capture(fn, min(L, K)), self._capture(fn, K % L) if K > L and K % L else None)
            except Exception as e:  # noqa: BLE001 - any capture failure falls back to launches
                print(f"bench: CUDA graph capture unavailable ({type(e).__name__}: {e}); stream launches",
                      file=sys.stderr)
                self.graph_ok = False
                torch.cuda.synchronize()
        soak_reps = 0
        if sampler is not None and soak_ms > 0 and gs is not None and est_ms:
            soak_reps = int(max(1, soak_ms / max(est_ms * min(L, K), 1e-3)))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()
        if sampler is not None:
            sampler.start()
            time.sleep(0.2)
        for _ in range(soak_reps):
            gs[0].replay()
        e0.record(self.stream)
        if gs is not None:
            for _ in range(K // L if K >= L else 1):
                gs[0].replay()
            if gs[1] is not None:
                gs[1].replay()
        else:
            for i in range(K):
                fn(i % R)
        e1.record(self.stream)
        torch.cuda.synchronize()
        if sampler is not None:
            sampler.clocks = sampler.stop()
            sampler.clocks["window"] = (f"{soak_reps * min(L, K)} untimed steps run back to back just before "
                                        f"the timed region, then the {K} timed steps")
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()
        return e0.elapsed_time(e1)

    def warm(self, ctx, n):
        import rank_bit_residual_b200 as rb
        for i in range(max(n, ctx["R"])):
            self.step(ctx, i)
        self.torch.cuda.synchronize()
        assert rb.svdq_check_status() == rb.SVDQ_OK

    # -- one record ----------------------------------------------------------
    def measure(self, ctx, K=None, warmup=3, sampler=None):
        """Time K steps (K None: enough for EXTRA_TIMED_MS), then each stage alone."""
        wl = ctx["wl"]
        B, M, N, r = wl.B, wl.M, wl.N, wl.rank
        R = ctx["R"]
        self.warm(ctx, warmup)
        # a first estimate of the step time sizes K and the soak
        est = self.time_calls(lambda i: self.step(ctx, i), 2 * R, R) / (2 * R)
        if K is None:
            K = int(min(4000, max(20, EXTRA_TIMED_MS / max(est, 1e-4))))
        total_ms = self.time_calls(lambda i: self.step(ctx, i), K, R, sampler=sampler, soak_ms=SOAK_MS,
                                   est_ms=est)
        Kg = int(min(2000, max(20, EXTRA_TIMED_MS / 2 / max(est, 1e-4))))
        gemm_ms = self.time_calls(lambda i: self.gemm_stage(ctx, i), Kg, R) / Kg
        act_ms = self.time_calls(lambda i: self.act_stage(ctx, i), Kg, R) / Kg
        import rank_bit_residual_b200 as rb
        assert rb.svdq_check_status() == rb.SVDQ_OK
        return {"K": K, "total_ms": total_ms, "gemm_ms": gemm_ms, "act_ms": act_ms, "Kg": Kg}


def roofline_of(wl, ms_per_step, gemm_ms, peaks, peak_src):
    """(step roofline dict, kernel roofline dict) of a measured workload."""
    B, M, N, r = wl.B, wl.M, wl.N, wl.rank
    ratio = 4.0 if wl.fmt != "int" else 2.0
    lowp_peak = ratio * peaks["bf16_tflops"]
    bytes_step = alg_bytes(B, M, N, r, wl.fmt, wl.bits, wl.bias is not None)
    ops_step = workload_ops(B, M, N, r)
    t_mem = bytes_step / (peaks["hbm_gbs"] * 1e9)
    t_cmp = (2.0 * B * M * N) / (lowp_peak * 1e12) + (2.0 * B * r * (M + N)) / (peaks["bf16_tflops"] * 1e12)
    t_rf = max(t_mem, t_cmp)
    step = {"t_roofline_us": t_rf * 1e6, "frac": t_rf / (ms_per_step * 1e-3), "alg_bytes": bytes_step,
            "ops": ops_step, "bound": "hbm" if t_mem >= t_cmp else "tensor"}
    if B <= 128:
        gb = gemm_alg_bytes(B, M, N, r, wl.fmt, wl.bits, wl.bias is not None)
        kern = ("gemv_kernel" if (wl.fmt == "int" and B <= 2) else "skinny_kernel") + "<" + (
            wl.fmt.upper() if wl.fmt != "int" else ("INT4 packed" if wl.bits <= 4 else "INT8")) + ">"
        ach = gb / (gemm_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": kern, "duration_us": gemm_ms * 1e3, "achieved": ach,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
                "alg_bytes_per_launch": gb, "peak_source": f"{peak_src} HBM copy bandwidth"}
    else:
        ach = gemm_alg_ops(B, M, N, r) / (gemm_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": f"gemm_pair_kernel<{wl.fmt.upper()}>", "duration_us": gemm_ms * 1e3,
                "achieved": ach, "peak": lowp_peak, "unit": "TFLOP/s", "frac": ach / lowp_peak,
                "alg_ops_per_launch": gemm_alg_ops(B, M, N, r),
                "peak_source": (f"{peak_src} bf16 GEMM burst x {ratio:g} "
                                f"(nominal {'fp4' if ratio == 4 else 'int8'}:bf16)")}
    return step, roof


def sampled_parity(ctx, y, rows_n=48):
    """Relative Frobenius and max errors of sampled rows of Y against the oracle
    evaluated on the prepared buffers of set 0."""
    import numpy as np
    import torch
    from oracle import codes as ocodes
    from oracle import prepared as oprep
    from oracle import nvfp4 as onv
    wl = ctx["wl"]
    w = ctx["sets"][0][0]
    B, M, N = wl.B, wl.M, wl.N
    rows = np.sort(np.random.default_rng(1).choice(B, size=min(B, rows_n), replace=False))
    ld = w.ld.float().cpu().numpy()[: w.rank_pad].T
    L2 = w.lu.float().cpu().numpy()[:, : w.rank_pad].T
    xr = np.asarray(wl.x[rows])
    if wl.fmt == "int":
        s_x = ocodes.int_scale_fp32(ocodes.act_max_fp32(wl.x, wl.scale), wl.bits)
        q, _, _ = ocodes.act_codes_int(xr, wl.scale, wl.bits, s=s_x)
        cw = w.codes.view(torch.int8).cpu().numpy().reshape(N, M)
        want = oprep.linear_int(xr, ld, L2, q, s_x, cw, float(w.w_scale[0].item()), wl.bias)
    elif wl.fmt == "mxfp4":
        from oracle import mxfp4 as omx
        ca, sa = omx.quantize(xr, div=wl.scale)
        cw = onv.unpack_nibbles(w.codes.cpu().numpy().reshape(N, M // 2))
        sfw = onv.sf_unswizzle(w.sf.cpu().numpy(), N, M // 32)
        want = oprep.linear_mxfp4(xr, ld, L2, ca, sa, cw, sfw, wl.bias)
    else:
        gx = onv.global_scale(ocodes.act_max_fp32(wl.x, wl.scale), "fp32")
        ca, sa, _ = onv.quantize(xr, gs=gx, div=wl.scale)
        cw = onv.unpack_nibbles(w.codes.cpu().numpy().reshape(N, M // 2))
        sfw = onv.sf_unswizzle(w.sf.cpu().numpy(), N, M // 16)
        want = oprep.linear_nvfp4(xr, ld, L2, ca, sa, gx, cw, sfw, float(w.w_scale[0].item()), wl.bias)
    got = y[torch.from_numpy(rows).to(y.device)].float().cpu().numpy()
    return {"rows_sampled": int(len(rows)), "rel_fro": float(np.linalg.norm(got - want) / np.linalg.norm(want)),
            "max_rel": float(np.max(np.abs(got - want)) / np.max(np.abs(want))), "y": "bf16 (rounding included)"}


def chain_record(eng, ctx, rows_list):
    """Consecutive linears of a square shape: layer k of a chain of R runs on set k's
    weights and reads layer k-1's Y, captured in one CUDA graph, plain and with each
    layer's activation pass a programmatic dependent of the previous GEMM."""
    import rank_bit_residual_b200 as rb
    torch = eng.torch
    R, sets, bias, x = ctx["R"], ctx["sets"], ctx["bias"], ctx["x"]

    def graph(pdl, rows):
        def run():
            prev = x[:rows]
            for k in range(R):
                wk, _, _, _, _, _, yk, wsk = sets[k]
                rb.svdq_linear(wk, prev, bias=bias, out=yk[:rows], workspace=wsk, pdl=pdl and k > 0)
                prev = yk[:rows]
        run()
        torch.cuda.synchronize()
        cap = torch.cuda.Stream()
        cap.wait_stream(eng.stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            run()
        eng.stream.wait_stream(cap)
        return g

    def timed(pdl, rows, reps):
        g = graph(pdl, rows)
        g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(eng.stream)
        for _ in range(reps):
            g.replay()
        e1.record(eng.stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / (reps * R)

    out = {"layers_per_chain": R, "note": "us per linear, chains of R layers of this shape captured in one "
                                          "CUDA graph; layer 0 plain in both"}
    for rows in rows_list:
        plain = timed(False, rows, 20)
        pdl = timed(True, rows, 20)
        out[f"B={rows}"] = {"plain_us": plain, "pdl_us": pdl, "saved_us": plain - pdl}
    assert rb.svdq_check_status() == rb.SVDQ_OK
    return out


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--rows", type=int, default=None, help="keep only the first rows of the workload's x")
    ap.add_argument("--configs", default=None, choices=["all", "none"],
                    help="per-configuration records (default: all for the default workload)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sets", type=int, default=0,
                    help="rotating buffer sets (default: enough to span three L2 sizes)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args, args.workload)
    configs = args.configs or ("all" if (args.workload == DEFAULT_WORKLOAD and args.rows is None) else "none")

    import numpy as np
    import torch
    import torch.distributed as dist

    import rank_bit_residual_b200 as rb

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    eng = Engine(dev, world, rank, local)
    peaks, peak_src = load_peaks()

    # ---------------------------------------------------------------- headline
    ctx = eng.setup(args.workload, rows=args.rows, nsets=args.sets)
    wl = ctx["wl"]
    B, M, N, r, R = wl.B, wl.M, wl.N, wl.rank, ctx["R"]
    sampler = ClockSampler(local)
    m = eng.measure(ctx, K=args.steps, warmup=args.warmup, sampler=sampler)
    K = m["K"]
    t = torch.tensor([m["total_ms"]], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    ops_step = workload_ops(B, M, N, r)
    value = world * K * ops_step / (total_ms * 1e-3) / 1e12
    ms_per_step = total_ms / K
    step_rf, roof = roofline_of(wl, ms_per_step, m["gemm_ms"], peaks, peak_src)
    roof["timing"] = "Kg launches back to back on rotating sets (CUDA graphs) between one CUDA event pair"
    csrc = os.path.join(ROOT, "rank_bit_residual_b200", "csrc")
    roof["traffic"] = read_profile_traffic(args.workload, [os.path.join(csrc, f) for f in
                                                           ("gemm_pair.cu", "gemm_common.cuh", "ptx.cuh")]) \
        if B > 128 else None

    # parity of the timed output (set 0 once more)
    eng.step(ctx, 0)
    torch.cuda.synchronize()
    parity = sampled_parity(ctx, ctx["sets"][0][6]) if rank == 0 else None

    # end to end through svdq_linear with host buffers: every step copies its x in
    # from pinned host memory and its Y out, on the rotating weights of the sets
    x_host = ctx["x"].cpu().pin_memory()
    y_host = torch.empty((B, N), dtype=torch.bfloat16).pin_memory()
    xd = torch.empty_like(ctx["x"])
    ye = torch.empty((B, N), dtype=torch.bfloat16, device=dev)
    ws = rb.LinearWorkspace()

    def e2e_step(i):
        xd.copy_(x_host, non_blocking=True)
        rb.svdq_linear(ctx["sets"][i % R][0], xd, bias=ctx["bias"], out=ye, workspace=ws)
        y_host.copy_(ye, non_blocking=True)

    Ke = max(3, min(50, K))
    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(eng.stream)
    for i in range(Ke):
        e2e_step(i)
    e1.record(eng.stream)
    torch.cuda.synchronize()
    e2e_ms = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(e2e_ms, op=dist.ReduceOp.MAX)
    e2e_value = world * Ke * ops_step / (float(e2e_ms.item()) * 1e-3) / 1e12

    out = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e2m1" if wl.fmt != "int" else "int8",
        "data": "synthetic",
        "config": config_of(wl, args.workload, {
            "l2": f"inputs larger than L2: {R} rotating buffer sets of {ctx['bytes_set'] / 1e6:.0f} MB",
            "launch": "CUDA graphs of many steps" if eng.graph_ok else "stream launches",
            "parallelism": f"replicas{world}"}),
        "gbs": step_rf["alg_bytes"] / (ms_per_step * 1e-3) / 1e9,
        "step_roofline": step_rf,
        "stages_ms": {"act": m["act_ms"], "gemm": m["gemm_ms"],
                      "note": "each stage alone, launched back to back on the rotating sets (CUDA "
                              "graphs of many launches between one event pair); in a step the GEMM "
                              "of a short batch overlaps the activation pass (dependent launch)"},
        "roofline": roof,
        "prepare_ms": ctx["prepare_ms"],
        "parity": parity,
        "e2e": {"value": e2e_value, "unit": "TOPS", "h2d_bytes_per_step": int(xd.numel() * xd.element_size()),
                "d2h_bytes_per_step": int(ye.numel() * ye.element_size()), "steps": Ke,
                "call": "svdq_linear (pinned host x -> device, Y -> pinned host), weights rotating over "
                        f"the {R} sets"},
        "gpu_launches": launches_per_step(wl) * K,
        "clocks": sampler.clocks,
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        v, dt, cores, sample = cpu_oracle_rate(wl)
        out["cpu_baseline"] = {"value": v, "unit": "TOPS", "cores": cores, "kind": "oracle",
                               "sample": sample, "seconds": dt}
    elif rank == 0:
        out["cpu_baseline"] = None
    del ctx

    # ------------------------------------------------------- other configurations
    if configs == "all" and world == 1:
        recs = []
        t_cfg = time.perf_counter()
        for name, rows in EXTRA_CONFIGS:
            print(f"bench: {name} rows={rows} at {time.perf_counter() - t_cfg:.1f} s", file=sys.stderr, flush=True)
            c = eng.setup(name, rows=rows)
            cw = c["wl"]
            mm = eng.measure(c)
            ms = mm["total_ms"] / mm["K"]
            srf, krf = roofline_of(cw, ms, mm["gemm_ms"], peaks, peak_src)
            rec = {"workload": name, "B": cw.B, "M": cw.M, "N": cw.N, "rank": cw.rank, "fmt": c["fmt"],
                   "us_per_step": ms * 1e3, "steps": mm["K"],
                   "tops": workload_ops(cw.B, cw.M, cw.N, cw.rank) / (ms * 1e-3) / 1e12,
                   "gbs": srf["alg_bytes"] / (ms * 1e-3) / 1e9,
                   "step_roofline": {"bound": srf["bound"], "t_roofline_us": srf["t_roofline_us"],
                                     "frac": srf["frac"]},
                   "kernel_roofline": {k: krf[k] for k in ("kernel", "bound", "duration_us", "achieved",
                                                           "unit", "peak", "frac")},
                   "act_us": mm["act_ms"] * 1e3, "gemm_us": mm["gemm_ms"] * 1e3,
                   "prepare_ms": c["prepare_ms"], "sets": c["R"], "launches_per_step": launches_per_step(cw)}
            eng.step(c, 0)
            torch.cuda.synchronize()
            rec["parity"] = sampled_parity(c, c["sets"][0][6], rows_n=16)
            if cw.M == cw.N and name.startswith("decode_") and rows in (1, 128):
                rec["chain"] = chain_record(eng, c, [rows])
            recs.append(rec)
            del c
        out["configs"] = recs
        out["configs_note"] = ("each record: its own rotating sets, CUDA-graph timing of back-to-back steps "
                               f"(~{EXTRA_TIMED_MS:.0f} ms), stages alone, prepare_ms = median time of "
                               "svdq_prepare for that weight (after the first call)")
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
