#!/usr/bin/env python3
"""Benchmark of the trellis-decode matmul hot path on B200.

Step = one forward pass of a seeded, synthetic trellis-coded layer stack
(RHT -> decode-GEMV for every phase of every layer) over one batch of tokens.
Default workload: the Qwen3-4B-shaped stack (36 layers) at batch 1; the
weights (codes + scales, 937 MB) stay resident in HBM, far larger than L2, so
no L2 flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                  [--workload qwen3-4b-m1|qwen3-4b-m512|llama-8b|27b] [--m M]

Prints ONE JSON line on rank 0.  N > 1 (torchrun) runs N independent replicas
(the path has no exchange step): value = all ranks' tokens / max-over-ranks time.
`--impl reference` times the CPU oracle (fp64 C, one host core) on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import tqsynth  # noqa: E402

PERSISTENT_MAX_M = 16  # tq_layer_stack runs one persistent kernel up to this many tokens
METRIC = "decode-GEMV compressed-weight GB/s (% of HBM peak); layer-stack tokens/s at batch 1"

WORKLOADS = {
    "qwen3-4b-m1": ("qwen3-4b-shaped", 1),
    "qwen3-4b-m512": ("qwen3-4b-shaped", 512),
    "llama-8b": ("llama-3.1-8b-shaped", 1),
    "27b": ("27b-class", 1),
}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


# ---- replicas (N > 1) ------------------------------------------------------------------

def max_over_ranks(x: float, dist, device) -> float:
    """The largest x over all ranks (every rank calls this in the same order);
    x itself when there is no process group."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(m: int, world: int, steps: int, ms_max: float) -> float:
    """Whole-job tokens/s of `world` independent replicas that each ran `steps`
    steps of m tokens, timed by the slowest rank (ms per step)."""
    return m * world * steps / (ms_max * steps * 1e-3)


# ---- clocks ----------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.nvml = []           # (time, SM MHz, max SM MHz, reason bits) from the polling thread
        self.window = None       # (t0, t1) of the timed region, time.perf_counter()
        self._stop = None
        self._thread = None

    def _poll_nvml(self):
        # NVML reads only (no setting is changed); ~1 ms between samples so that
        # a timed region of a few tens of ms still gets many
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            while not self._stop.is_set():
                self.nvml.append((time.perf_counter(), pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), mx,
                                  reasons(h)))
                time.sleep(0.001)
            pynvml.nvmlShutdown()
        except Exception:  # no NVML: the nvidia-smi samples stand
            pass

    def mark(self, t0: float, t1: float):
        """The timed region (time.perf_counter() before its first launch and
        after its synchronize)."""
        self.window = (t0, t1)

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._poll_nvml, daemon=True)
        self._thread.start()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    # NVML clock-event reason bits
    NVML_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}

    def summary(self):
        if self.window is not None:
            t0, t1 = self.window
            inside = [x for x in self.nvml if t0 <= x[0] <= t1]
            if inside:
                reasons = sorted(n for n, bit in self.NVML_BITS.items() if any(x[3] & bit for x in inside))
                return {"sm_mhz": float(np.median([x[1] for x in inside])), "sm_max_mhz": float(inside[0][2]),
                        "reasons": reasons, "samples": len(inside), "source": "nvml, timed region"}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "source": "nvidia-smi"}


# ---- stack construction ----------------------------------------------------------

def build_stack(tq, shape, seed, device):
    import torch
    cb_host = tqsynth.codebook(seed)
    cbd = torch.from_numpy(cb_host.view(np.int16)).to(device)
    layers = []
    for l in range(shape.layers):
        w = {}
        for i, (op, n, k) in enumerate(shape.ops()):
            codes = tqsynth.codes(seed, l, i, n, k)
            scales = tqsynth.scales(seed, l, i, n, k)
            w[op] = tq.DeviceWeight.from_host(codes, scales, cbd, n, k, device=device)
        layers.append(w)
    return layers


def phase_bytes(shape, m):
    """Algorithmic bytes of each of the 4 phases of one layer: packed weights
    (codes + scales) + codebook + activations in (bf16) + outputs (fp32 y and
    bf16 handoff)."""
    ops = {op: (n, k) for op, n, k in shape.ops()}
    groups = (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))
    out = []
    for p, g in enumerate(groups):
        k = ops[g[0]][1]
        packed = sum(tqsynth.pack_bytes(*ops[op]) for op in g)
        n_tot = sum(ops[op][0] for op in g)
        out.append(packed + 16384 + m * k * 2 + m * n_tot * 4 + m * ops[g[0]][0] * 2)
    return out


def ncu_traffic(shape_name, layers, m):
    """DRAM bytes (read + write) per launch of the batch-1 stack kernel, from the
    committed ncu summary of the Qwen3-4B-shaped stack (measured on 6 layers,
    scaled per layer); None for any other shape or batch (not captured)."""
    p = os.path.join(ROOT, "profiles", "stack1_kernel_qwen3-4b-shaped_m1.md")
    if m != 1 or shape_name != "qwen3-4b-shaped" or not os.path.exists(p):
        return None
    with open(p) as f:
        for ln in f:
            if ln.startswith("dram_bytes_per_layer:"):
                return float(ln.split(":")[1]) * layers
    return None


# ---- reference arm (CPU oracle) ---------------------------------------------------

def run_reference(args, shape, m):
    import oracle
    oracle.build()
    seed = 0
    steps, warm = args.steps, args.warmup
    # per-step CPU budget so that warmup + steps end in about two minutes
    budget = max(2.0, 120.0 / max(1, steps + warm))
    ops = shape.ops()
    x = tqsynth.activations(seed, m, shape.hidden)
    cb = tqsynth.codebook(seed)
    # rows of each op in the sample: the same fraction f of every op of layer 0
    t0 = time.perf_counter()
    probe_rows = 4
    for i, (op, n, k) in enumerate(ops):
        c = tqsynth.codes_rows(seed, 0, i, k, 0, probe_rows)
        s = tqsynth.scales(seed, 0, i, probe_rows, k)
        xr = np.zeros((m, k))
        oracle.linear_rows(c, s, cb, k, xr, m, 0, probe_rows)
    per_row_layer = (time.perf_counter() - t0) / probe_rows  # one row of every op
    rows = max(1, min(min(n for _, n, _ in ops), int(budget / max(per_row_layer, 1e-9))))
    frac = {op: rows / n for op, n, _ in ops}

    def one_step():
        h = x
        ts = time.perf_counter()
        for p, group in enumerate(oracle.PHASES):
            k = dict((o, kk) for o, _, kk in ops)[group[0]]
            xr = oracle.rht(h if h.shape[1] == k else tqsynth.activations(seed + 1 + p, m, k), m, k,
                            oracle.stack_phase_seed(seed, 0, p))
            for op in group:
                i = [o for o, _, _ in ops].index(op)
                n = [nn for o, nn, _ in ops if o == op][0]
                r = max(1, int(round(frac[op] * n)))
                c = tqsynth.codes_rows(seed, 0, i, k, 0, r)
                s = tqsynth.scales(seed, 0, i, r, k)
                oracle.linear_rows(c, s, cb, k, xr, m, 0, r)
        return time.perf_counter() - ts

    for _ in range(warm):
        one_step()
    times = [one_step() for _ in range(steps)]
    t_step = float(np.mean(times))
    # the sample is `rows` rows of every op of one layer: scale to the whole stack
    full_rows = sum(n for _, n, _ in ops)
    sample_rows = sum(max(1, int(round(frac[op] * n))) for op, n, _ in ops)
    t_token = t_step * (full_rows / sample_rows) * shape.layers / m
    value = 1.0 / t_token
    sample = (f"{sample_rows} of {full_rows} weight rows of layer 0 (all 7 ops, all 4 RHTs) at m={m}, "
              f"scaled by rows and by {shape.layers} layers")
    cpu = {"value": value, "unit": "tok/s", "cores": 1, "kind": "oracle", "sample": sample}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": warm, "ms_per_step": t_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{shape.name} stack, {shape.layers} layers, batch {m}", "layers": shape.layers,
                       "batch": m, "parallelism": "replicas"},
            "cpu_baseline": cpu, "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0,
                                         "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---- our arm ------------------------------------------------------------------------

def cpu_baseline_quick(shape, m):
    """The oracle on ~10-20 s of host work: the same fraction of the rows of
    each op of layer 0 (with its RHT), each op's time scaled by its row count,
    summed, and scaled to the whole stack."""
    import oracle
    oracle.build()
    seed = 0
    cb = tqsynth.codebook(seed)
    ops = shape.ops()
    t_target = 12.0
    cost = []  # seconds per row of each op (2-row probe)
    for i, (op, n, k) in enumerate(ops):
        c = tqsynth.codes_rows(seed, 0, i, k, 0, 2)
        s = tqsynth.scales(seed, 0, i, 2, k)
        t0 = time.perf_counter()
        oracle.linear_rows(c, s, cb, k, np.zeros((m, k)), m, 0, 2)
        cost.append((time.perf_counter() - t0) / 2)
    t_est = sum(n * c for (_, n, _), c in zip(ops, cost))  # one whole layer
    frac = min(1.0, t_target / max(t_est, 1e-9))
    n_layers = max(1, min(shape.layers, int(round(t_target / max(t_est, 1e-9))))) if frac >= 1.0 else 1
    x = tqsynth.activations(seed, m, shape.hidden)
    t_layers, t_all, done = 0.0, 0.0, 0
    for l in range(n_layers):
        for i, (op, n, k) in enumerate(ops):
            rows = max(1, min(n, int(round(frac * n))))
            xin = x if k == shape.hidden else tqsynth.activations(seed + 1 + i, m, k)
            c = tqsynth.codes_rows(seed, l, i, k, 0, rows)
            s = tqsynth.scales(seed, l, i, rows, k)
            ts = time.perf_counter()
            xr = oracle.rht(xin, m, k, oracle.stack_phase_seed(seed, l, 0))
            oracle.linear_rows(c, s, cb, k, xr, m, 0, rows)
            t = time.perf_counter() - ts
            t_all += t
            t_layers += t * n / rows
            done += rows
    full_rows = sum(n for _, n, _ in ops)
    t_token = t_layers / n_layers * shape.layers / m
    what = (f"all {full_rows} rows of layers 0-{n_layers - 1}" if frac >= 1.0 else
            f"{done} of the {full_rows} rows of layer 0 (the same fraction of each of its 7 ops)")
    return {"value": 1.0 / t_token, "unit": "tok/s", "cores": 1, "kind": "oracle",
            "sample": f"{what} with their RHTs, m={m}, {t_all:.1f} s single-threaded, each op scaled by its "
                      f"row count, then to {shape.layers} layers"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="qwen3-4b-m1", choices=sorted(WORKLOADS))
    ap.add_argument("--m", type=int, default=None)
    ap.add_argument("--layers", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    stack_name, m = WORKLOADS[args.workload]
    if args.m is not None:
        m = args.m
    shape = tqsynth.stack_shape(stack_name, args.layers)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, shape, m)
        return

    import torch
    import decode_matmul_b200 as tq

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    layers = build_stack(tq, shape, 0, dev)
    structs = [tq.layer_struct(L) for L in layers]
    sargs = tq.StackArgs(structs, m)
    ws = tq.workspace(tq.tq_layer_stack_workspace(structs, m), dev)
    h_in = torch.from_numpy(tqsynth.activations(0, m, shape.hidden).view(np.int16)).to(dev)
    h_out = torch.empty_like(h_in)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    # one step = tq_layer_stack over the whole stack; captured once in a CUDA graph
    with torch.cuda.stream(stream):
        tq.tq_layer_stack(sargs, h_in, 0, h_out, ws, stream=stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        tq.tq_layer_stack(sargs, h_in, 0, h_out, ws, stream=stream)
    torch.cuda.synchronize()

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        time.sleep(0.3)  # sampler start-up
        t_start = time.perf_counter()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
        stream.synchronize()
        clk.mark(t_start, time.perf_counter())
    torch.cuda.synchronize()
    barrier()
    ms = e0.elapsed_time(e1) / args.steps
    ms_max = max_over_ranks(ms, dist, dev)

    # per-phase kernel durations (eager, events between launches) for the roofline
    pb = phase_bytes(shape, m)
    ph_ms = [0.0] * 4
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    reps = max(1, min(args.steps, 5))
    ph_seed = [tq.tq_stack_phase_seed(0, 0, p) for p in range(4)]
    ysz = max(sum(n for op, n, _ in shape.ops() if op in g) for g in (("q", "k", "v"), ("o",), ("gate", "up"), ("down",)))
    ybuf = torch.empty((m, ysz), dtype=torch.float32, device=dev)
    bufs = {0: torch.empty((m, shape.q_dim), dtype=torch.int16, device=dev),
            1: torch.empty((m, shape.hidden), dtype=torch.int16, device=dev),
            2: torch.empty((m, shape.inter), dtype=torch.int16, device=dev),
            3: torch.empty((m, shape.hidden), dtype=torch.int16, device=dev)}
    wsp = tq.workspace(max(tq.tq_layer_phase_workspace(structs[0], p, m) for p in range(4)), dev)
    ins = [h_in, bufs[0], bufs[1], bufs[2]]
    with torch.cuda.stream(stream):
        for r in range(reps + 1):
            for l in range(shape.layers):
                ev[0].record(stream)
                for p in range(4):
                    tq.tq_layer_phase(structs[l], p, ins[p], ph_seed[p], ybuf, bufs[p], wsp, stream=stream)
                    ev[p + 1].record(stream)
                if r > 0 and l % 6 == 0:
                    ev[4].synchronize()
                    for p in range(4):
                        ph_ms[p] += ev[p].elapsed_time(ev[p + 1])
    stream.synchronize()
    nsamp = reps * len(range(0, shape.layers, 6))
    ph_ms = [t / nsamp for t in ph_ms]
    hbm, tflops, peak_src = measured_peaks()
    bytes_step_layer = sum(pb)
    kern_ms_layer = sum(ph_ms)
    flops_layer = 2.0 * m * shape.weights_per_layer()
    tensor_tflops = flops_layer / (kern_ms_layer * 1e-3) / 1e12
    # up to 16 tokens the timed step is one launch of a persistent stack kernel
    # (plus a 256-byte memset of its barrier word), so its duration is the step time
    stack_bytes = bytes_step_layer * shape.layers
    achieved = stack_bytes / (ms * 1e-3) / 1e9
    value = replica_throughput(m, world, args.steps, ms_max)

    # end to end through the C ABI with host buffers: pinned h_in -> device,
    # tq_layer_stack (direct call, no graph), result -> pinned host
    h_host = torch.from_numpy(tqsynth.activations(1, m, shape.hidden).view(np.int16)).pin_memory()
    o_host = torch.empty_like(h_host).pin_memory()
    d_in = torch.empty_like(h_in)
    ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for i in range(args.warmup + args.steps):
            if i == args.warmup:
                stream.synchronize()
                barrier()
                ee0.record(stream)
            d_in.copy_(h_host, non_blocking=True)
            tq.tq_layer_stack(sargs, d_in, 0, h_out, ws, stream=stream)
            o_host.copy_(h_out, non_blocking=True)
        ee1.record(stream)
    stream.synchronize()
    e2e_ms = ee0.elapsed_time(ee1) / args.steps
    e2e_val = replica_throughput(m, world, 1, max_over_ranks(e2e_ms, dist, dev))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_quick(shape, m)

    if dist is not None:
        del graph
        dist.destroy_process_group()

    if rank != 0:
        return
    bytes_token = shape.packed_bytes() / m
    line = {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic: seeded random codes/scales/codebook/activations",
        "config": {"workload": f"{shape.name} stack, {shape.layers} layers, batch {m}", "layers": shape.layers,
                   "batch": m, "hidden": shape.hidden, "inter": shape.inter, "seed": 0,
                   "packed_bytes": shape.packed_bytes(), "parallelism": f"replicas x{world}",
                   "l2": "no flush: 937 MB-5.6 GB of resident weights per step exceed the 126 MB L2"},
        "compressed_weight_gbs": bytes_token * value / world / 1e9,
        "hbm_frac_of_measured": bytes_token * value / world / 1e9 / hbm,
        "roofline": ({"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                      "frac": achieved / hbm, "traffic": ncu_traffic(shape.name, shape.layers, m),
                      "peak_source": peak_src,
                      "kernel": ("stack1_kernel (persistent: RHT + decode + mma.sync, every phase of every layer)"
                                 if m == 1 else
                                 "stackn_kernel (persistent: grid-split RHT + decode + mma.sync, every phase of "
                                 "every layer)"),
                      "bytes_per_launch": stack_bytes,
                      "eager_phase_ms": ph_ms, "phase_bytes": pb} if m <= PERSISTENT_MAX_M else
                     {"bound": "hbm", "achieved": bytes_step_layer / (kern_ms_layer * 1e-3) / 1e9, "peak": hbm,
                      "unit": "GB/s", "frac": bytes_step_layer / (kern_ms_layer * 1e-3) / 1e9 / hbm,
                      "traffic": None, "peak_source": peak_src,
                      "kernel": "rht_kernel + dmma_kernel (mma.sync register decode), all 4 phases",
                      "phase_ms": ph_ms, "phase_bytes": pb} if m < 32 else
                     {"bound": "tensor", "achieved": tensor_tflops, "peak": tflops, "unit": "TFLOP/s",
                      "frac": tensor_tflops / tflops, "traffic": None, "peak_source": peak_src,
                      "kernel": "rht_kernel + umma_kernel (tcgen05 decode-to-smem GEMM), all 4 phases",
                      "phase_ms": ph_ms, "phase_flops": [2.0 * m * sum(n * k for o, n, k in shape.ops() if o in g)
                                                         for g in (("q", "k", "v"), ("o",), ("gate", "up"),
                                                                   ("down",))]}),
        "clocks": clk.summary(),
        "e2e": {"value": e2e_val, "unit": "tok/s", "h2d_bytes_per_step": int(h_host.numel() * 2),
                "d2h_bytes_per_step": int(o_host.numel() * 2)},
        "gpu_launches": args.steps * (1 if m <= PERSISTENT_MAX_M else 4 * shape.layers * 2),
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
