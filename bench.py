#!/usr/bin/env python3
"""Benchmark of the 8-bit quantized linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl q8|reference]
                    [--workload NAME] [--no-extras]

A step is one forward of the quantized linear layer on one batch of synthetic
input: dynamic per-token activation quantization followed by the W8A8 GEMM
with its dequant epilogue (weights are quantized once, offline, before the
timed region, as the pages do on load).  The default workload is the
q_proj-shaped decode layer: 16 tokens x 4096 -> 4096, bf16 in, asymmetric
uint8 weights, INT32 accumulation, bf16 out.

Timing: W warm-up steps, then exactly K steps replayed from CUDA graphs,
bracketed by a barrier and a device synchronize, timed with CUDA events on the
launching stream, max over ranks.  Steps rotate over 16 independent weight
sets (268 MB of codes, more than the 126 MB L2), so every step reads its
weights from HBM.  Prints one JSON line on rank 0.

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
ROTATE = 16           # independent layers cycled through by the timed steps
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

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
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


# ---------------------------------------------------------------- inputs

def decode_layers(q8, dev, rotate: int, seed0: int):
    """Rotating decode layers drawn with the decode recipe on the device:
    W ~ N(0, 0.02) with 1% of entries redrawn from N(0, 0.2), X ~ N(0, 1)."""
    w = workloads.WORKLOADS["decode_q_proj"]
    g = torch.Generator(device=dev)
    layers = []
    for i in range(rotate):
        g.manual_seed(seed0 + i)
        X = torch.randn(w.m, w.k, generator=g, device=dev).to(torch.bfloat16)
        W = torch.randn(w.n, w.k, generator=g, device=dev) * 0.02
        heavy = torch.rand(w.n, w.k, generator=g, device=dev) < 0.01
        W = torch.where(heavy, torch.randn(w.n, w.k, generator=g, device=dev) * 0.2, W)
        W = W.to(torch.bfloat16)
        qw = q8.q8_quantize_weight(W, "asym", "u8")
        del W
        qa = q8.QAct(torch.empty((w.m, w.k), dtype=torch.int8, device=dev),
                     torch.empty(w.m, dtype=torch.float32, device=dev),
                     torch.empty(w.m, dtype=torch.int32, device=dev), q8.Q8_S8)
        Y = torch.empty((w.m, w.n), dtype=torch.bfloat16, device=dev)
        layers.append({"X": X, "qw": qw, "qa": qa, "Y": Y})
    torch.cuda.synchronize()
    return layers


def decode_gemm_bytes(w):
    """Algorithmic HBM bytes of one decode GEMM launch: weight codes, activation
    codes, bf16 output, per-channel scale/zero point, per-token scale/row sum."""
    return w.n * w.k + w.m * w.k + 2 * w.m * w.n + 8 * w.n + 8 * w.m


# ---------------------------------------------------------------- q8 arm

def run_q8(args, world, rank, local):
    from bit_quantized_b200 import q8
    dev = torch.device("cuda", local)
    wl = workloads.WORKLOADS["decode_q_proj"]
    pk = peaks()
    ops_per_step = 2.0 * wl.m * wl.n * wl.k
    layers = decode_layers(q8, dev, ROTATE, seed0=1000 * (rank + 1))

    def step(i):
        L = layers[i % ROTATE]
        q8.q8_quantize_act(L["X"], "int8", out=L["qa"])
        q8.q8_linear_w8a8(L["qa"], L["qw"], out=L["Y"])

    def gemm_only(i):
        L = layers[i % ROTATE]
        q8.q8_linear_w8a8(L["qa"], L["qw"], out=L["Y"])

    # warm-up (eager, through the public API)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # One CUDA graph per rotation of the 16 layers (no event nodes inside: an
    # event record node costs several microseconds, more than a decode kernel).
    def make_graphs(fn):
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for i in range(ROTATE):
                fn(i)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        out = {}
        for n_steps in sorted({ROTATE, args.steps % ROTATE} - {0}):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(n_steps):
                    fn(i)
            out[n_steps] = g
        return out

    def timed(gmap, sampler=None):
        full, rem = divmod(args.steps, ROTATE)
        for _ in range(max(1, args.warmup // ROTATE)):
            gmap[ROTATE].replay()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        if sampler:
            sampler.start()
            time.sleep(0.25)
        t0.record()
        for _ in range(full):
            gmap[ROTATE].replay()
        if rem:
            gmap[rem].replay()
        t1.record()
        torch.cuda.synchronize()
        clk = sampler.stop() if sampler else None
        barrier(world)
        return max_over_ranks(t0.elapsed_time(t1), world), clk

    step_graphs = make_graphs(step)
    sampler = ClockSampler(local)
    ms_max, clocks = timed(step_graphs, sampler)
    value = args.steps * world * ops_per_step / (ms_max * 1e-3) / 1e12
    # The dominant kernel's average launch duration: the same K launches of the
    # GEMM alone, replayed the same way right after, CUDA events on this stream.
    gemm_graphs = make_graphs(gemm_only)
    gemm_ms, _ = timed(gemm_graphs)
    gemm_avg_ms = gemm_ms / args.steps
    del step_graphs, gemm_graphs

    # e2e: pinned host input -> C ABI calls -> pinned host output, every step
    e2e = run_e2e(q8, layers, args, world, ops_per_step)

    algo_bytes = decode_gemm_bytes(wl)
    achieved = algo_bytes / (gemm_avg_ms * 1e-3) / 1e9
    traffic = load_profile_traffic("decode_gemm")
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "s8",
        "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) weights with 1% N(0,0.2) tail)",
        "config": {"workload": "decode_q_proj", "m_tokens": wl.m, "n_out": wl.n, "k_in": wl.k,
                   "x_dtype": "bf16", "weight": "per-channel asymmetric uint8 + fp32 S/Z",
                   "activation": "per-token symmetric int8", "accumulate": "int32",
                   "out": "bf16", "parallelism": f"dp{world} (independent batches per GPU)",
                   "l2": f"steps rotate over {ROTATE} weight sets "
                         f"({ROTATE * wl.n * wl.k / 1e6:.0f} MB of codes > 126 MB L2)",
                   "timing": "CUDA graphs of 16 steps, CUDA events, max over ranks"},
        "roofline": {"bound": "hbm", "kernel": "gemm_decode_kernel<16, s8xu8>",
                     "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": traffic,
                     "algorithmic_bytes": algo_bytes, "avg_launch_us": round(gemm_avg_ms * 1e3, 3),
                     "duration_from": "K GEMM launches replayed alone right after the timed steps",
                     "peak_source": pk["source"] + " (MEASURED_PEAKS.json hbm_gbs, burst copy)"},
        "e2e": e2e,
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds)
    if world == 1 and rank == 0 and not args.no_extras:
        line["per_config"] = extras(q8, dev, pk)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(q8, layers, args, world, ops_per_step):
    w = workloads.WORKLOADS["decode_q_proj"]
    steps = min(args.steps, args.e2e_steps)
    hx = [L["X"].cpu().pin_memory() for L in layers]
    hy = [torch.empty((w.m, w.n), dtype=torch.bfloat16).pin_memory() for _ in layers]
    dx = torch.empty_like(layers[0]["X"])
    for i in range(min(args.warmup, 8)):
        L = layers[i % ROTATE]
        dx.copy_(hx[i % ROTATE], non_blocking=True)
        q8.q8_quantize_act(dx, "int8", out=L["qa"])
        q8.q8_linear_w8a8(L["qa"], L["qw"], out=L["Y"])
        hy[i % ROTATE].copy_(L["Y"], non_blocking=True)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    t0.record()
    for i in range(steps):
        L = layers[i % ROTATE]
        dx.copy_(hx[i % ROTATE], non_blocking=True)
        q8.q8_quantize_act(dx, "int8", out=L["qa"])
        q8.q8_linear_w8a8(L["qa"], L["qw"], out=L["Y"])
        hy[i % ROTATE].copy_(L["Y"], non_blocking=True)
    t1.record()
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1), world)
    return {"value": round(steps * world * ops_per_step / (ms * 1e-3) / 1e12, 3), "unit": UNIT,
            "h2d_bytes_per_step": int(hx[0].numel() * hx[0].element_size()),
            "d2h_bytes_per_step": int(hy[0].numel() * hy[0].element_size()),
            "steps": steps, "ms_per_step": ms / steps, "wall_s": round(wall, 4),
            "path": "pinned host X -> q8_quantize_act -> q8_linear_w8a8 -> pinned host Y, eager"}


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


def source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_quantized_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
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


def extras(q8, dev, pk):
    """Kernel-level numbers for every workload (single GPU, L2 flushed per launch)."""
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    int8_peak = pk["bf16_tflops"] * NOMINAL_INT8_OVER_BF16
    out = {"int8_fp8_peak_tops": int8_peak,
           "peak_note": f"{pk['source']} bf16 burst {pk['bf16_tflops']} TFLOP/s x 2 (nominal "
                        "dense INT8/FP8 : bf16 ratio 4.5 : 2.25)",
           "hbm_peak_gbs": pk["hbm_gbs"]}
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
            r["launches_per_call"] = 5
        else:
            scheme = "int8" if w.kind == "w8a8_int8" else "fp8"
            qa = q8.q8_quantize_act(Xd, scheme, clip_ub=w.clip_ub)
            t_act = _time_kernel(lambda: q8.q8_quantize_act(Xd, scheme, clip_ub=w.clip_ub, out=qa), flush)
            act_bytes = w.m * w.k * (2 + 1) + 8 * w.m
            r["act_quant_us"] = round(t_act * 1e3, 2)
            r["act_quant_gbs"] = round(act_bytes / (t_act * 1e-3) / 1e9, 1)
            r["act_quant_frac_hbm"] = round(act_bytes / (t_act * 1e-3) / 1e9 / pk["hbm_gbs"], 3)
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
            if name == "prefill_ffn_up":
                wq_bytes = w.n * w.k * 3 + 8 * w.n
                t_w = _time_kernel(lambda: q8.q8_quantize_weight(Wd, w.weight_scheme, w.weight_codes), flush, reps=5)
                r["weight_quant_us"] = round(t_w * 1e3, 1)
                r["weight_quant_gbs"] = round(wq_bytes / (t_w * 1e-3) / 1e9, 1)
        out[name] = r
        del Xd, Wd
    torch.cuda.synchronize()
    return out


# ---------------------------------------------------------------- CPU oracle

def oracle_decode_inputs():
    from oracle import oracle as O
    X, W, _ = workloads.make_inputs("decode_q_proj")
    x32 = O.widen16(workloads.bits16(X), "bf16")
    w32 = O.widen16(workloads.bits16(W), "bf16")
    wq, Sw, Zw = O.quant_weight(w32, "asym", "u8")
    return O, x32, wq, Sw, Zw


def cpu_baseline(seconds: float = 10.0):
    """The oracle, as it stands, on full decode steps for about `seconds`."""
    O, x32, wq, Sw, Zw = oracle_decode_inputs()
    w = workloads.WORKLOADS["decode_q_proj"]
    ops = 2.0 * w.m * w.n * w.k
    done, t0 = 0, time.perf_counter()
    while True:
        xq, Sx, rs = O.quant_act_int8(x32)
        O.linear_w8a8_int8(xq, Sx, rs, wq, Sw, Zw)
        done += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": round(done * ops / dt / 1e12, 6), "unit": UNIT, "cores": O.threads(),
            "kind": "oracle",
            "sample": f"{done} full decode steps (16x4096 act quant + 16x4096x4096 int8 GEMM "
                      f"+ epilogue) in {dt:.1f} s; weight quantization excluded as on the GPU"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    O, x32, wq, Sw, Zw = oracle_decode_inputs()
    w = workloads.WORKLOADS["decode_q_proj"]
    # Size each step's sample so that warm-up + K steps take about a minute.
    t0 = time.perf_counter()
    xq, Sx, rs = O.quant_act_int8(x32[:1])
    O.linear_w8a8_int8(xq, Sx, rs, wq, Sw, Zw, None, np.array([0]), np.arange(w.n))
    per_col = (time.perf_counter() - t0) / w.n
    budget = 60.0 / max(1, args.steps + args.warmup)
    cols = int(max(16, min(w.n, budget / max(per_col, 1e-9))))
    colsel = np.arange(cols)
    rows = np.array([0])

    def step(i):
        r = np.array([i % w.m])
        xq, Sx, rs = O.quant_act_int8(x32[r])
        O.linear_w8a8_int8(xq, Sx, rs, wq, Sw, Zw, None, np.array([0]), colsel)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    ops = 2.0 * rows.size * cols * w.k * args.steps
    value = ops / dt / 1e12
    sample = (f"each step: 1 token row of the 16x4096 decode input (act quant) x {cols} of 4096 "
              "output columns (int8 GEMM + epilogue)")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "s8", "data": "synthetic",
            "config": {"workload": "decode_q_proj", "m_tokens": w.m, "n_out": w.n, "k_in": w.k},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": O.threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=32)
    ap.add_argument("--impl", choices=["q8", "reference"], default="q8")
    ap.add_argument("--e2e-steps", type=int, default=20000)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
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
