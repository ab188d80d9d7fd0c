#!/usr/bin/env python3
"""Benchmark of the 8-bit quantized linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl q8|reference]
                    [--workload NAME] [--no-extras] [--no-cpu-baseline]

A step is one forward of the quantized linear layer on one batch of synthetic
input: dynamic per-token activation quantization followed by the W8A8 GEMM
with its dequant epilogue (weights are quantized once, offline, before the
timed region, as the pages do on load).  The default workload is the largest
one, the FBGEMM-style FP8 rowwise linear: 4096 tokens x 8192 -> 8192, bf16 in,
per-token e4m3 activations with the 1200 upper bound, per-channel e4m3
weights, fp32 accumulation, bf16 out; --workload picks another of the seeded
workloads in workloads.py (decode and prefill INT8, LLM.int8), and the
per_config extras time every workload's kernels one launch at a time.

The roofline entry divides by the dense tensor peak for the GEMM's own dtype:
the measured bf16 peak (MEASURED_PEAKS.json) times the nominal INT8/FP8 : bf16
ratio of 2, burst or sustained according to the length of the timed region,
and also by the INT8 and FP8 throughput of the library GEMMs
(torch._int_mm, torch._scaled_mm) measured at 8192^3 in the same run.

Timing: W warm-up steps, then exactly K steps replayed from CUDA graphs,
bracketed by a barrier and a device synchronize, timed with CUDA events on the
launching stream, max over ranks.  Steps rotate over independent layers
whose working set is more than twice the 126 MB L2 (16 layers, 268 MB of
weight codes, for the decode layer), so every step reads its weights from
HBM.  Prints one JSON line on rank 0.

--impl reference times the CPU oracle (oracle/) on the host cores instead,
each step a bounded sample of the same workload.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "W8A8 linear TOPS & % of B200 INT8/FP8 tensor peak; act-quant GB/s vs HBM"
UNIT = "TOPS"
NOMINAL_INT8_OVER_BF16 = 2.0   # dense INT8/FP8 4.5 P vs bf16 2.25 P per GPU


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---------------------------------------------------------------- distributed

def dist_setup(n_gpus: int, backend: str | None = None):
    """One process per GPU: reads RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* from
    the environment (torchrun) and joins the process group (NCCL on GPUs)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def aggregate_tops(steps: int, world: int, ops_per_step: float, ms_max: float) -> float:
    """Whole-job throughput: the operations of every rank's K steps over the
    slowest rank's time (weak scaling: per-GPU work fixed as N grows)."""
    return steps * world * ops_per_step / (ms_max * 1e-3) / 1e12


def max_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- workloads

# Default timed steps per workload (about a second or two of device time each).
DEFAULT_STEPS = {"decode_q_proj": 100000, "tiny_mixed": 50000, "mixed_512": 20000,
                 "prefill_ffn_up": 4000, "fp8_rowwise": 2000}
DEFAULT_E2E_STEPS = {"decode_q_proj": 20000, "tiny_mixed": 20000, "mixed_512": 2000,
                     "prefill_ffn_up": 100, "fp8_rowwise": 50}
L2_BYTES = 126 * 1024 * 1024


def step_hbm_bytes(w) -> int:
    """Bytes one step must move: weight codes, bf16/fp16 input, activation codes, bf16 output."""
    return w.n * w.k + 2 * w.m * w.k + w.m * w.k + 2 * w.m * w.n


def rotation(w) -> int:
    """Independent layers cycled through so the working set exceeds twice the L2."""
    r = -(-2 * L2_BYTES // step_hbm_bytes(w))
    return int(min(16, max(2, r)))


def make_layers(q8, dev, name: str, rotate: int, seed0: int):
    """`rotate` independent layers of the workload, drawn with its seeded recipe
    (workloads.make_inputs, one seed per layer), weights quantized once."""
    w = workloads.WORKLOADS[name]
    layers = []
    for i in range(rotate):
        X, W, _ = workloads.make_inputs(name, seed=seed0 + i)
        X, Wd = X.to(dev), W.to(dev)
        qw = q8.q8_quantize_weight(Wd, w.weight_scheme, w.weight_codes)
        del Wd
        L = {"X": X, "qw": qw, "Y": torch.empty((w.m, w.n), dtype=torch.bfloat16, device=dev)}
        if w.kind == "w8a8_int8":
            L["qa"] = q8.QAct(torch.empty((w.m, w.k), dtype=torch.int8, device=dev),
                              torch.empty(w.m, dtype=torch.float32, device=dev),
                              torch.empty(w.m, dtype=torch.int32, device=dev), q8.Q8_S8)
        elif w.kind == "w8a8_fp8":
            L["qa"] = q8.QAct(torch.empty((w.m, w.k), dtype=torch.float8_e4m3fn, device=dev),
                              torch.empty(w.m, dtype=torch.float32, device=dev), None, q8.Q8_E4M3)
        else:
            L["ws"] = torch.empty(q8.q8_workspace_size(q8.Q8_OP_LINEAR_INT8_MIXED, w.m, w.n, w.k),
                                  dtype=torch.uint8, device=dev)
        layers.append(L)
    torch.cuda.synchronize()
    return layers


def step_functions(q8, w):
    """(step, dominant kernel alone, kernel launches per step) for a workload."""
    if w.kind == "int8_mixed":
        def step(L, X=None):
            q8.q8_linear_int8_mixed(L["X"] if X is None else X, L["qw"], w.threshold,
                                    out=L["Y"], workspace=L["ws"])
        return step, step, 3
    scheme = "int8" if w.kind == "w8a8_int8" else "fp8"

    def step(L, X=None):
        # activation quantization + linear in one call (two launches; the GEMM's
        # prologue and weight loads overlap the quantizer)
        q8.q8_linear_w8a8_dynamic(L["X"] if X is None else X, L["qw"], scheme,
                                  clip_ub=w.clip_ub, out=L["Y"], act=L["qa"])

    def gemm(L, X=None):
        q8.q8_linear_w8a8(L["qa"], L["qw"], out=L["Y"])
    return step, gemm, 2


# A timed region shorter than this runs at the burst clocks of a GPU that has
# not yet settled under its power cap; longer ones at the sustained clocks.
SUSTAINED_REGION_MS = 1000.0


def dominant_kernel(w, gemm_ms: float, region_ms: float, pk: dict, lib_peaks: dict):
    """Roofline entry of the step's dominant kernel (the GEMM)."""
    ops = 2.0 * w.m * w.n * w.k
    t = gemm_ms * 1e-3
    algo_bytes = w.n * w.k + w.m * w.k + 2 * w.m * w.n + 8 * w.n + 8 * w.m
    if w.m <= 64:
        achieved = algo_bytes / t / 1e9
        return {"bound": "hbm", "kernel": "gemm_decode_kernel (split-K cluster)",
                "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm_gbs"], 4), "algorithmic_bytes": algo_bytes,
                "peak_source": pk["source"] + " hbm_gbs (MEASURED_PEAKS.json, copy)"}
    sustained = region_ms >= SUSTAINED_REGION_MS
    bf16 = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
    peak = bf16 * NOMINAL_INT8_OVER_BF16
    achieved = ops / t / 1e12
    if w.kind == "int8_mixed":
        kernel = ("gemm_pair_kernel (LLM.int8, cta_group::2, int32 + fp32 accumulators)" if w.m > 128
                  else "gemm_tile_kernel (LLM.int8, int32 + fp32 accumulators)")
    elif w.m > 256:
        kernel = "gemm_pair_kernel (cta_group::2, 256-row tiles on SM pairs)"
    else:
        kernel = "gemm_tile_kernel (128-row tiles)"
    out = {"bound": "tensor", "kernel": kernel,
           "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
           "frac": round(achieved / peak, 4), "algorithmic_ops": ops,
           "peak_source": (f"{pk['source']} bf16 {'sustained' if sustained else 'burst'} {bf16} x 2 "
                           "(nominal dense INT8/FP8 : bf16 = 4.5 : 2.25); the kernel's timed region "
                           f"lasted {region_ms:.1f} ms ({'>=' if sustained else '<'} "
                           f"{SUSTAINED_REGION_MS:.0f} ms)")}
    lib_key = "fp8_tops" if w.kind == "w8a8_fp8" else "int8_tops"
    lp = lib_peaks.get(lib_key)
    if lp:
        out["peak_library"] = lp
        out["frac_of_library"] = round(achieved / lp, 4)
        out["library_source"] = lib_peaks.get(lib_key.replace("_tops", "_how"))
    return out


def library_peaks(dev) -> dict:
    """Dense INT8 and FP8 GEMM throughput of the library kernels at 8192^3 on
    this GPU: torch._int_mm (int8 x int8 -> int32) and torch._scaled_mm (e4m3 x
    e4m3 -> bf16, rowwise fp32 scales where supported, else per-tensor).  Best
    of 10 launches after 3 warm-ups, CUDA events.  Reported next to the
    derived peak; a call the installed torch does not support is left out."""
    n = 8192
    out = {"shape": f"{n}^3", "how": "best of 10 launches, CUDA events"}
    g = torch.Generator(device=dev).manual_seed(0)

    def best(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(10):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return 2.0 * n ** 3 / (min(ts) * 1e-3) / 1e12

    try:
        A = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=g)
        B = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=g)
        out["int8_tops"] = round(best(lambda: torch._int_mm(A, B.t())), 1)
        out["int8_how"] = "torch._int_mm int8 8192^3 (B column-major)"
        del A, B
    except Exception as e:  # noqa: BLE001 - report, do not fail the bench
        out["int8_error"] = f"{type(e).__name__}: {str(e)[:120]}"
    try:
        A = (torch.randn(n, n, device=dev, generator=g) * 4).to(torch.float8_e4m3fn)
        B = (torch.randn(n, n, device=dev, generator=g) * 4).to(torch.float8_e4m3fn)
        sa = torch.ones((n, 1), dtype=torch.float32, device=dev)
        sb = torch.ones((1, n), dtype=torch.float32, device=dev)
        try:
            fn = lambda: torch._scaled_mm(A, B.t(), scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16)
            fn()
            out["fp8_how"] = "torch._scaled_mm e4m3 8192^3, rowwise scales, bf16 out"
        except Exception:  # noqa: BLE001 - rowwise scaling unsupported: per-tensor
            one = torch.ones((), dtype=torch.float32, device=dev)
            fn = lambda: torch._scaled_mm(A, B.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            out["fp8_how"] = "torch._scaled_mm e4m3 8192^3, per-tensor scales, bf16 out"
        out["fp8_tops"] = round(best(fn), 1)
        del A, B
    except Exception as e:  # noqa: BLE001
        out["fp8_error"] = f"{type(e).__name__}: {str(e)[:120]}"
    torch.cuda.synchronize()
    return out


def launch_spread(fn, layers, R, n: int) -> dict:
    """Median, p10 and p90 of n single launches of fn (CUDA events around each,
    layers rotated as in the timed region)."""
    for i in range(3):
        fn(layers[i % R])
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    for i in range(n):
        ev[i][0].record()
        fn(layers[i % R])
        ev[i][1].record()
    torch.cuda.synchronize()
    ts = np.array([a.elapsed_time(b) * 1e3 for a, b in ev])
    return {"median_us": round(float(np.median(ts)), 3), "p10_us": round(float(np.percentile(ts, 10)), 3),
            "p90_us": round(float(np.percentile(ts, 90)), 3), "launches": n,
            "how": "one launch between CUDA events, eager, layers rotated"}


def describe(w):
    if w.kind == "w8a8_fp8":
        return {"x_dtype": "bf16", "weight": "per-channel FP8 e4m3 + fp32 scale",
                "activation": f"per-token FP8 e4m3, clip {w.clip_ub}", "accumulate": "fp32",
                "out": "bf16"}
    wt = {"asym": "per-channel asymmetric " + ("uint8" if w.weight_codes == "u8" else "int8")
          + " + fp32 S/Z", "sym": "per-channel symmetric int8 + fp32 S"}[w.weight_scheme]
    d = {"x_dtype": "fp16" if w.x_dtype == torch.float16 else "bf16", "weight": wt,
         "activation": "per-token symmetric int8", "accumulate": "int32", "out": "bf16"}
    if w.kind == "int8_mixed":
        d["outliers"] = f"LLM.int8 threshold {w.threshold}, fp16 outlier GEMM merged"
    return d


# ---------------------------------------------------------------- q8 arm

def run_q8(args, world, rank, local):
    from bit_quantized_b200 import q8
    dev = torch.device("cuda", local)
    wl = workloads.WORKLOADS[args.workload]
    pk = peaks()
    ops_per_step = 2.0 * wl.m * wl.n * wl.k
    R = rotation(wl)
    layers = make_layers(q8, dev, args.workload, R, seed0=1000 * rank)
    step_fn, kernel_fn, launches = step_functions(q8, wl)

    # warm-up (eager, through the public API)
    for i in range(args.warmup):
        step_fn(layers[i % R])
    torch.cuda.synchronize()

    # One CUDA graph per rotation of the R layers (no event nodes inside: an
    # event record node costs several microseconds, more than a decode kernel).
    def make_graphs(fn):
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for i in range(R):
                fn(layers[i])
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        out = {}
        for n_steps in sorted({R, args.steps % R} - {0}):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(n_steps):
                    fn(layers[i])
            out[n_steps] = g
        return out

    def timed(gmap, sampler=None):
        full, rem = divmod(args.steps, R)
        for _ in range(max(1, args.warmup // R)):
            gmap[R].replay()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        if sampler:
            sampler.start()
            time.sleep(0.25)
        t0.record()
        for _ in range(full):
            gmap[R].replay()
        if rem:
            gmap[rem].replay()
        t1.record()
        torch.cuda.synchronize()
        clk = sampler.stop() if sampler else None
        barrier(world)
        return max_over_ranks(t0.elapsed_time(t1), world), clk

    step_graphs = make_graphs(step_fn)
    ms_max, clocks = timed(step_graphs, ClockSampler(local))
    value = aggregate_tops(args.steps, world, ops_per_step, ms_max)
    del step_graphs
    # The dominant kernel's average launch duration: the same K launches of the
    # GEMM alone (for LLM.int8, the whole call), replayed the same way right
    # after the timed steps, CUDA events on this stream.
    kernel_graphs = make_graphs(kernel_fn)
    kernel_ms, _ = timed(kernel_graphs)
    kernel_avg_ms = kernel_ms / args.steps
    del kernel_graphs

    spread = launch_spread(kernel_fn, layers, R, n=min(max(args.steps, 20), 200))
    e2e = run_e2e(q8, layers, R, step_fn, args, world, ops_per_step, wl)
    lib_peaks = library_peaks(dev) if (world == 1 and not args.no_library_peaks) else {}
    roof = dominant_kernel(wl, kernel_avg_ms, kernel_ms, pk, lib_peaks)
    roof["launch_spread"] = spread
    roof["traffic"] = load_profile_traffic(args.workload)
    roof["avg_launch_us"] = round(kernel_avg_ms * 1e3, 3)
    roof["duration_from"] = ("K launches of the kernel replayed alone right after the timed steps"
                             if launches == 2 else "K whole calls replayed right after the timed steps")
    ws_bytes = R * step_hbm_bytes(wl)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if wl.kind == "w8a8_fp8" else "s8",
        "data": "synthetic (seeded recipe of workloads.py, one seed per rotated layer)",
        "config": {"workload": args.workload, "m_tokens": wl.m, "n_out": wl.n, "k_in": wl.k,
                   **describe(wl), "parallelism": f"dp{world} (independent batches per GPU)",
                   "l2": (f"steps rotate over {R} layers ({ws_bytes / 1e6:.0f} MB > 126 MB L2)"
                          if ws_bytes > L2_BYTES else
                          f"{R} layers ({ws_bytes / 1e6:.1f} MB) stay L2-resident")},
        "timing": f"CUDA graphs of {R} steps, CUDA events, max over ranks",
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": launches * args.steps,
        "clocks": clocks,
        "library_peaks": lib_peaks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, seconds=args.cpu_seconds)
    if world == 1 and rank == 0 and not args.no_extras:
        line["per_config"] = extras(q8, dev, pk)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(q8, layers, R, step_fn, args, world, ops_per_step, w):
    """Same step through the public API with the input copied from pinned host
    memory and the bf16 output copied back to pinned host memory every step.

    The steps are replayed as a CUDA graph of S steps (a multiple of the R
    layers, up to 16), as a serving loop would issue them: each step's
    host-to-device copy runs on a copy stream and may overlap earlier steps'
    compute and output copies, the step's call runs on the compute stream once
    its input has landed, and the device-to-host copy of its result on a third
    stream.  Step i uses layer i mod R; a copy into a layer's input buffer
    waits until the step that last read it has finished, and a step waits
    until the previous output copy of its layer has left the device.  Every
    step still moves its own input and output; a replay ends only when the
    last step's output is on the host."""
    S = R * max(1, min(args.steps, args.e2e_steps, 16) // R)
    reps = max(1, min(args.steps, args.e2e_steps) // S)
    steps = reps * S
    hx = [L["X"].cpu().pin_memory() for L in layers]
    hy = [torch.empty((w.m, w.n), dtype=torch.bfloat16).pin_memory() for _ in layers]
    dx = [torch.empty_like(L["X"]) for L in layers]
    s_main, s_in, s_comp, s_out = (torch.cuda.Stream() for _ in range(4))
    ev_in = [torch.cuda.Event() for _ in range(S)]
    ev_done = [torch.cuda.Event() for _ in range(S)]
    ev_out = [torch.cuda.Event() for _ in range(S)]

    def record_steps():
        fork = torch.cuda.Event()
        fork.record(s_main)
        for st in (s_in, s_comp, s_out):
            st.wait_event(fork)
        for i in range(S):
            j = i % R
            with torch.cuda.stream(s_in):
                if i >= R:
                    s_in.wait_event(ev_done[i - R])      # dx[j] read by step i - R
                dx[j].copy_(hx[j], non_blocking=True)
                ev_in[i].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[i])
                if i >= R:
                    s_comp.wait_event(ev_out[i - R])     # Y of layer j copied out
                step_fn(layers[j], dx[j])
                ev_done[i].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i])
                hy[j].copy_(layers[j]["Y"], non_blocking=True)
                ev_out[i].record(s_out)
        for st in (s_in, s_comp, s_out):
            s_main.wait_stream(st)

    with torch.cuda.stream(s_main):
        record_steps()                 # eager warm-up of every call
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s_main):
        record_steps()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    with torch.cuda.stream(s_main):
        t0.record(s_main)
        for _ in range(reps):
            g.replay()
        t1.record(s_main)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1), world)
    ok = all(torch.equal(hy[i], layers[i]["Y"].cpu()) for i in range(R))
    del g
    return {"value": round(steps * world * ops_per_step / (ms * 1e-3) / 1e12, 3), "unit": UNIT,
            "h2d_bytes_per_step": int(hx[0].numel() * hx[0].element_size()),
            "d2h_bytes_per_step": int(hy[0].numel() * hy[0].element_size()),
            "steps": steps, "ms_per_step": ms / steps, "wall_s": round(wall, 4),
            "host_output_matches_device": ok,
            "path": "pinned host X -> H2D copy stream -> q8_linear_w8a8_dynamic / q8_linear_int8_mixed "
                    "(C ABI) on a compute stream -> D2H copy stream -> pinned host Y; CUDA graph of "
                    f"{S} steps over {R} layers, a step's copies overlap other steps' compute and copies"}


def load_profile_traffic(kernel_tag: str):
    """DRAM bytes per launch recorded from an ncu capture of the current kernels
    (profiles/traffic.json), or None when no capture matches them."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    entry = t.get(kernel_tag)
    if not entry:
        return None
    src = entry.get("source_hash")
    if src and src != source_hash():
        return None
    return entry.get("dram_bytes_per_launch")


# Sources the GEMM kernels are compiled from (a traffic entry stays valid
# while these are unchanged).
GEMM_SOURCES = ("q8_device.cuh", "q8_gemm.cu", "q8_qmath.cuh")


def source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_quantized_b200", "csrc")
    for f in GEMM_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------- per-config extras

def _time_kernel(fn, flush, reps=20):
    """Median CUDA-event time of fn() with L2 flushed before every launch."""
    ts = []
    for _ in range(reps + 3):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts[3:])


def _time_graph(fn, count: int, reps: int = 5) -> float:
    """Average time (ms) of one fn(i) call, i = 0..count-1 captured back to
    back in a CUDA graph and replayed `reps` times (no host launch overhead
    between the calls; the rotated inputs keep them reading from HBM)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(count):
            fn(i)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(count):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / (reps * count)
    del g
    return ms


def _rotated_copies(X, min_bytes: int):
    """Independent copies of X whose total exceeds min_bytes (at least 2)."""
    per = X.numel() * X.element_size()
    n = int(max(2, min(16, -(-min_bytes // per))))
    return [X.clone() for _ in range(n)]


def extras(q8, dev, pk):
    """Kernel-level numbers for every workload (single GPU, L2 flushed per launch)."""
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    int8_peak = pk["bf16_tflops"] * NOMINAL_INT8_OVER_BF16
    out = {"int8_fp8_peak_tops": int8_peak,
           "peak_note": f"{pk['source']} bf16 burst {pk['bf16_tflops']} TFLOP/s x 2 (nominal "
                        "dense INT8/FP8 : bf16 ratio 4.5 : 2.25)",
           "hbm_peak_gbs": pk["hbm_gbs"],
           "timing": "each figure: one launch between CUDA events right after an L2 flush (launch "
                     "latency included; the graph-replayed step above is the sustained figure)"}
    for name in workloads.ORDER:
        w = workloads.WORKLOADS[name]
        X, W, _ = workloads.make_inputs(name)
        Xd, Wd = X.to(dev), W.to(dev)
        r = {}
        if w.kind == "int8_mixed":
            qw = q8.q8_quantize_weight(Wd, w.weight_scheme, w.weight_codes)
            Y = torch.empty((w.m, w.n), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(q8.q8_workspace_size(1, w.m, w.n, w.k), dtype=torch.uint8, device=dev)
            t = _time_kernel(lambda: q8.q8_linear_int8_mixed(Xd, qw, w.threshold, out=Y,
                                                             workspace=ws), flush)
            r["mixed_call_us"] = round(t * 1e3, 2)
            r["tops"] = round(2.0 * w.m * w.n * w.k / (t * 1e-3) / 1e12, 2)
            r["launches_per_call"] = 3
        else:
            scheme = "int8" if w.kind == "w8a8_int8" else "fp8"
            qa = q8.q8_quantize_act(Xd, scheme, clip_ub=w.clip_ub)
            t_act = _time_kernel(lambda: q8.q8_quantize_act(Xd, scheme, clip_ub=w.clip_ub, out=qa), flush)
            act_bytes = w.m * w.k * (2 + 1) + 8 * w.m
            r["act_quant_us"] = round(t_act * 1e3, 2)
            r["act_quant_gbs"] = round(act_bytes / (t_act * 1e-3) / 1e9, 1)
            r["act_quant_frac_hbm"] = round(act_bytes / (t_act * 1e-3) / 1e9 / pk["hbm_gbs"], 3)
            # The same quantizer back to back over rotated inputs (> 2 x L2) in a
            # CUDA graph: the kernel's own bandwidth, without launch overhead.
            xs = _rotated_copies(Xd, 2 * L2_BYTES)
            qas = [q8.q8_quantize_act(x, scheme, clip_ub=w.clip_ub) for x in xs]
            t_g = _time_graph(lambda i: q8.q8_quantize_act(xs[i], scheme, clip_ub=w.clip_ub, out=qas[i]),
                              len(xs))
            r["act_quant_graph_us"] = round(t_g * 1e3, 2)
            r["act_quant_graph_gbs"] = round(act_bytes / (t_g * 1e-3) / 1e9, 1)
            r["act_quant_graph_frac_hbm"] = round(act_bytes / (t_g * 1e-3) / 1e9 / pk["hbm_gbs"], 3)
            del xs, qas
            qw = q8.q8_quantize_weight(Wd, w.weight_scheme, w.weight_codes)
            Y = torch.empty((w.m, w.n), dtype=torch.bfloat16, device=dev)
            t = _time_kernel(lambda: q8.q8_linear_w8a8(qa, qw, out=Y), flush)
            tops = 2.0 * w.m * w.n * w.k / (t * 1e-3) / 1e12
            gbytes = (w.m * w.k + w.n * w.k + 2 * w.m * w.n) / (t * 1e-3) / 1e9
            r["gemm_us"] = round(t * 1e3, 2)
            r["gemm_tops"] = round(tops, 1)
            r["gemm_frac_tensor_peak"] = round(tops / int8_peak, 4)
            r["gemm_gbs"] = round(gbytes, 1)
            r["gemm_frac_hbm"] = round(gbytes / pk["hbm_gbs"], 4)
            if name in ("prefill_ffn_up", "fp8_rowwise"):
                wq_bytes = w.n * w.k * 3 + 8 * w.n
                t_w = _time_kernel(lambda: q8.q8_quantize_weight(Wd, w.weight_scheme, w.weight_codes), flush, reps=5)
                r["weight_quant_us"] = round(t_w * 1e3, 1)
                r["weight_quant_gbs"] = round(wq_bytes / (t_w * 1e-3) / 1e9, 1)
                r["weight_quant_frac_hbm"] = round(wq_bytes / (t_w * 1e-3) / 1e9 / pk["hbm_gbs"], 3)
            if w.kind == "w8a8_int8":
                # Static scales (calibrated once; here 1.1 x the batch absmax / 127) and the
                # linear that re-quantizes its output to INT8 for the next layer.
                S = float(1.1 * float(Xd.float().abs().max()) / 127)
                qs = q8.q8_quantize_act_static(Xd, S)
                t_s = _time_kernel(lambda: q8.q8_quantize_act_static(Xd, S, out=qs), flush)
                r["static_act_quant_us"] = round(t_s * 1e3, 2)
                r["static_act_quant_gbs"] = round(act_bytes / (t_s * 1e-3) / 1e9, 1)
                mult = torch.rand(w.k, generator=torch.Generator().manual_seed(1)).add_(0.5).to(dev)
                qm = q8.q8_quantize_act_smooth(Xd, mult)
                t_m = _time_kernel(lambda: q8.q8_quantize_act_smooth(Xd, mult, out=qm), flush)
                r["smooth_act_quant_us"] = round(t_m * 1e3, 2)
                r["smooth_act_quant_gbs"] = round(act_bytes / (t_m * 1e-3) / 1e9, 1)
                So = float(1.2 * float(q8.q8_linear_w8a8(qs, qw).float().abs().max()) / 127)
                Yq = torch.empty((w.m, w.n), dtype=torch.int8, device=dev)
                t_r = _time_kernel(lambda: q8.q8_linear_w8a8_requant(qs, qw, So, out=Yq), flush)
                r["requant_gemm_us"] = round(t_r * 1e3, 2)
                r["requant_gemm_tops"] = round(2.0 * w.m * w.n * w.k / (t_r * 1e-3) / 1e12, 1)
                # Group-wise 4-bit weights (groups of 128 along K) with the same
                # bf16 activations: codes k/2 bytes per row + fp32 scales, X, Y.
                g4 = q8.q8_quantize_weight_g4(Wd, 128)
                Y4 = torch.empty((w.m, w.n), dtype=torch.bfloat16, device=dev)
                t_4 = _time_kernel(lambda: q8.q8_linear_w4a16(Xd, g4, out=Y4), flush)
                b4 = w.n * w.k // 2 + 4 * w.n * (w.k // 128) + 2 * w.m * w.k + 2 * w.m * w.n
                r["w4a16_us"] = round(t_4 * 1e3, 2)
                r["w4a16_tflops"] = round(2.0 * w.m * w.n * w.k / (t_4 * 1e-3) / 1e12, 1)
                r["w4a16_gbs"] = round(b4 / (t_4 * 1e-3) / 1e9, 1)
                r["w4a16_frac_hbm"] = round(b4 / (t_4 * 1e-3) / 1e9 / pk["hbm_gbs"], 4)
                r["w4a16_frac_bf16_peak"] = round(2.0 * w.m * w.n * w.k / (t_4 * 1e-3) / 1e12
                                                  / pk["bf16_tflops"], 4)
        out[name] = r
        del Xd, Wd
    out["moe_fp8_grouped"] = moe_extra(q8, dev, pk, flush)
    torch.cuda.synchronize()
    return out


def moe_extra(q8, dev, pk, flush):
    """Grouped FP8 rowwise linear of a mixture-of-experts layer: 16 experts of
    2048 x 4096 (e4m3 weights, 134 MB, beyond L2) and 4096 tokens, each routed
    to a seeded uniformly drawn expert."""
    E, n, k, m = 16, 2048, 4096, 4096
    g = torch.Generator().manual_seed(5)
    pick = torch.randint(0, E, (m,), generator=g)
    counts = torch.bincount(pick, minlength=E)
    off = torch.zeros(E + 1, dtype=torch.int32)
    off[1:] = torch.cumsum(counts, 0).to(torch.int32)
    X = workloads.random_matrix(m, k, torch.bfloat16, 6).to(dev)
    W = workloads.random_matrix(E * n, k, torch.bfloat16, 7, 0.02).to(dev)
    qa = q8.q8_quantize_act(X, "fp8", clip_ub=1200.0)
    qw = q8.q8_quantize_weight(W, "fp8", "e4m3")
    del W
    offd = off.to(dev)
    Y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    t = _time_kernel(lambda: q8.q8_linear_fp8_grouped(qa, qw, E, offd, out=Y), flush)
    tops = 2.0 * m * n * k / (t * 1e-3) / 1e12
    int8_peak = pk["bf16_tflops"] * NOMINAL_INT8_OVER_BF16
    return {"shape": f"{E} experts x {n} x {k}, {m} tokens (max {int(counts.max())}, "
                     f"min {int(counts.min())} per expert)",
            "grouped_us": round(t * 1e3, 2), "grouped_tops": round(tops, 1),
            "grouped_frac_fp8_peak": round(tops / int8_peak, 4),
            "grouped_gbs": round((m * k + E * n * k + 2 * m * n) / (t * 1e-3) / 1e9, 1)}


# ---------------------------------------------------------------- CPU oracle

def oracle_inputs(name: str):
    from oracle import oracle as O
    w = workloads.WORKLOADS[name]
    X, W, _ = workloads.make_inputs(name)
    fmt = "f16" if w.x_dtype == torch.float16 else "bf16"
    x32 = O.widen16(workloads.bits16(X), fmt)
    w32 = O.widen16(workloads.bits16(W), fmt)
    q = O.quant_weight(w32, w.weight_scheme, w.weight_codes)
    return O, w, x32, q


def oracle_step(O, w, x32, q, rows, cols):
    """One oracle forward of the workload on the given token rows and output columns."""
    wq, Sw, Zw = q
    xs = x32[rows]
    r = np.arange(len(rows))
    if w.kind == "w8a8_int8":
        xq, Sx, rs = O.quant_act_int8(xs)
        O.linear_w8a8_int8(xq, Sx, rs, wq, Sw, Zw, None, r, cols)
    elif w.kind == "w8a8_fp8":
        xq, Sx = O.quant_act_fp8(xs, w.clip_ub)
        O.linear_w8a8_fp8(xq, Sx, wq, Sw, None, r, cols)
    else:
        O.linear_int8_mixed(x32, wq, Sw, Zw, w.threshold, rows=rows, cols=cols)


def cpu_baseline(name: str, seconds: float = 10.0):
    """The oracle, as it stands, on the workload's step for about `seconds`:
    full steps when one takes under a second, else steps on a row sample."""
    O, w, x32, q = oracle_inputs(name)
    cols = np.arange(w.n)
    threads = O.threads()
    # The oracle runs its rows on parallel threads: time a step of one row per
    # thread, then size the sample so one step takes about a second.
    t0 = time.perf_counter()
    oracle_step(O, w, x32, q, np.arange(min(w.m, threads)), cols)
    per_round = time.perf_counter() - t0
    rounds = int(max(1, 1.0 / max(per_round, 1e-9)))
    rows_n = int(min(w.m, threads * rounds))
    rows = np.arange(rows_n)
    ops = 2.0 * rows_n * w.n * w.k
    done, t0 = 0, time.perf_counter()
    while True:
        oracle_step(O, w, x32, q, rows, cols)
        done += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    what = "full steps" if rows_n == w.m else f"steps on {rows_n} of {w.m} token rows"
    cores = min(threads, rows_n)
    # The same work on one host thread, for a quarter of the time, on a row
    # sample a thread's share of the step (so that one step stays short).
    rows1 = rows[:max(1, rows_n // max(cores, 1))]
    ops1 = 2.0 * len(rows1) * w.n * w.k
    O.set_threads(1)
    try:
        done1, t1 = 0, time.perf_counter()
        while True:
            oracle_step(O, w, x32, q, rows1, cols)
            done1 += 1
            if time.perf_counter() - t1 >= seconds / 4:
                break
        dt1 = time.perf_counter() - t1
    finally:
        O.set_threads(threads)
    return {"value": round(done * ops / dt / 1e12, 6), "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": f"{done} {what} of {name} ({w.m}x{w.n}x{w.k}: activation quantization + "
                      f"GEMM + epilogue) in {dt:.1f} s on {cores} threads; weight quantization "
                      "excluded as on the GPU",
            "one_thread": {"value": round(done1 * ops1 / dt1 / 1e12, 6), "unit": UNIT,
                           "sample": f"{done1} steps on {len(rows1)} token rows in {dt1:.1f} s "
                                     "on 1 thread"}}


def run_reference(args, world, rank):
    if rank != 0:
        return
    O, w, x32, q = oracle_inputs(args.workload)
    cols_all = np.arange(w.n)
    # Each step's sample: one token row per host thread (the oracle runs rows
    # on parallel threads) x as many output columns as keep warm-up + K steps
    # within about a minute.
    threads = O.threads()
    nrows = min(w.m, threads)
    t0 = time.perf_counter()
    oracle_step(O, w, x32, q, np.arange(nrows), cols_all)
    per_col = (time.perf_counter() - t0) / w.n
    budget = 60.0 / max(1, args.steps + args.warmup)
    ncols = int(max(16, min(w.n, budget / max(per_col, 1e-9))))
    cols = cols_all[:ncols]

    def step(i):
        oracle_step(O, w, x32, q, (np.arange(nrows) + i * nrows) % w.m, cols)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    value = 2.0 * nrows * ncols * w.k * args.steps / dt / 1e12
    sample = (f"each step: {nrows} token rows of the {w.m}x{w.k} {args.workload} input (activation "
              f"quantization) x {ncols} of {w.n} output columns (GEMM + epilogue), one row per "
              "host thread")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3" if w.kind == "w8a8_fp8" else "s8",
            "data": "synthetic",
            "config": {"workload": args.workload, "m_tokens": w.m, "n_out": w.n, "k_in": w.k,
                       **describe(w), "parallelism": f"dp{world} (independent batches per GPU)"},
            "timing": "host wall clock of the oracle on the host cores, bounded sample per step",
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": nrows,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile(args):
    """One kernel of a workload, a few launches, for an ncu capture of a
    small case: 3 warm-up launches, then --steps launches; prints one line
    with the median launch time (CUDA events)."""
    from bit_quantized_b200 import q8
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workloads.WORKLOADS[args.workload]
    X, W, _ = workloads.make_inputs(args.workload)
    Xd, Wd = X.to(dev), W.to(dev)
    scheme = "fp8" if w.kind == "w8a8_fp8" else "int8"
    fn = None
    if args.profile == "moe":
        E, n, k, m = 16, 2048, 4096, 4096
        g = torch.Generator().manual_seed(5)
        counts = torch.bincount(torch.randint(0, E, (m,), generator=g), minlength=E)
        off = torch.zeros(E + 1, dtype=torch.int32)
        off[1:] = torch.cumsum(counts, 0).to(torch.int32)
        qa = q8.q8_quantize_act(workloads.random_matrix(m, k, torch.bfloat16, 6).to(dev), "fp8", clip_ub=1200.0)
        qw = q8.q8_quantize_weight(workloads.random_matrix(E * n, k, torch.bfloat16, 7, 0.02).to(dev), "fp8", "e4m3")
        offd, Y = off.to(dev), torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        fn = lambda: q8.q8_linear_fp8_grouped(qa, qw, E, offd, out=Y)
    elif args.profile == "weight_quant":
        fn = lambda: q8.q8_quantize_weight(Wd, w.weight_scheme, w.weight_codes)
    elif w.kind == "int8_mixed":
        qw = q8.q8_quantize_weight(Wd, w.weight_scheme, w.weight_codes)
        Y = torch.empty((w.m, w.n), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(q8.q8_workspace_size(q8.Q8_OP_LINEAR_INT8_MIXED, w.m, w.n, w.k),
                         dtype=torch.uint8, device=dev)
        fn = lambda: q8.q8_linear_int8_mixed(Xd, qw, w.threshold, out=Y, workspace=ws)
    else:
        qw = q8.q8_quantize_weight(Wd, w.weight_scheme, w.weight_codes)
        qa = q8.q8_quantize_act(Xd, scheme, clip_ub=w.clip_ub)
        Y = torch.empty((w.m, w.n), dtype=torch.bfloat16, device=dev)
        if args.profile == "act_quant":
            fn = lambda: q8.q8_quantize_act(Xd, scheme, clip_ub=w.clip_ub, out=qa)
        elif args.profile == "gemm":
            fn = lambda: q8.q8_linear_w8a8(qa, qw, out=Y)
        else:
            fn = lambda: q8.q8_linear_w8a8_dynamic(Xd, qw, scheme, clip_ub=w.clip_ub, out=Y, act=qa)
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) * 1e3)
    print(json.dumps({"profile": args.profile, "workload": args.workload, "launches": args.steps,
                      "median_us": round(float(np.median(ts)), 2)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=32)
    ap.add_argument("--impl", choices=["q8", "reference"], default="q8")
    ap.add_argument("--workload", choices=workloads.ORDER, default="fp8_rowwise")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-library-peaks", action="store_true")
    ap.add_argument("--profile", choices=["gemm", "step", "act_quant", "weight_quant", "moe"],
                    default=None, help="run one kernel of the workload a few times (for ncu)")
    args = ap.parse_args()
    if args.profile is not None:
        args.steps = 3 if args.steps is None else args.steps
        run_profile(args)
        return
    if args.steps is None:
        args.steps = DEFAULT_STEPS[args.workload]
    if args.e2e_steps is None:
        args.e2e_steps = DEFAULT_E2E_STEPS[args.workload]
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    run_q8(args, world, rank, local)


if __name__ == "__main__":
    main()
