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
The line also carries `gemv`: the batch-1 decode-GEMV alone (tq_gemv on a
32768 x 16384 weight, two copies read in turn so no launch finds its weight in
L2), the first half of the metric, with its own roofline and clocks.
`--impl reference` times the CPU oracle (fp64 C, on all host cores) on a
bounded sample of the same workload; our arm's `cpu_baseline` is the same
recipe, on all cores and on one.
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
REGISTER_DECODE_MAX_M = 32  # up to this many tokens the phases use the register-decode kernel, tcgen05 above
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


STACK_SOURCES = ("tq_common.cuh", "tq_rht.cuh", "tq_dmma.cuh", "tq_stack1.cuh")


def kernel_source_hash(names=STACK_SOURCES) -> str:
    """sha256 over the CUDA sources of a kernel (to tell whether an ncu figure
    was taken on the kernel that runs now)."""
    import hashlib
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "decode_matmul_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def ncu_traffic(shape_name, layers, m):
    """DRAM bytes (read + write) per launch of the batch-1 stack kernel from
    the ncu figure stored in profiles/ (measured on a few layers, scaled by
    layers: every layer has the same shapes), or None when there is no figure
    for this shape and batch or the kernel's sources changed since it was
    taken."""
    p = os.path.join(ROOT, "profiles", "stack1_kernel_traffic.json")
    if m != 1 or not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("workload") != shape_name or d.get("source_sha256") != kernel_source_hash():
        return None
    return float(d["dram_bytes_per_layer"]) * layers


# ---- the CPU oracle on a bounded sample (reference arm and cpu_baseline) ---------------

def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def oracle_layer_sample(shape, m, frac, threads, layer=0, seed=0):
    """One layer of the stack on the oracle, sampled: per phase one RHT of a
    seeded bf16 input of the phase's width with that layer's phase seed, then
    the first round(frac * n) rows of every op of the phase (decode + fp64
    matmul), split over `threads` host threads (the C oracle releases the GIL).
    Returns (seconds spent, the same scaled to every row of the layer, rows
    done)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    cb = tqsynth.codebook(seed)
    ops = shape.ops()
    opi = {op: i for i, (op, _, _) in enumerate(ops)}
    dims = {op: (n, k) for op, n, k in ops}
    t_all = t_full = 0.0
    done = 0
    with ThreadPoolExecutor(max_workers=threads) as ex:
        for p, group in enumerate(oracle.PHASES):
            k = dims[group[0]][1]
            x = tqsynth.activations(seed, m, k, stream=p + 1)
            data = []
            for op in group:
                n = dims[op][0]
                r = max(1, min(n, int(round(frac * n))))
                data.append((op, n, r, tqsynth.codes_rows(seed, layer, opi[op], k, 0, r),
                             tqsynth.scales(seed, layer, opi[op], r, k)))
            ts = time.perf_counter()
            xr = oracle.rht(x, m, k, oracle.stack_phase_seed(seed, layer, p))
            t_rht = time.perf_counter() - ts
            t_phase_full = t_rht
            for op, n, r, c, sc in data:
                ts = time.perf_counter()
                chunks = [(i * r // threads, (i + 1) * r // threads) for i in range(threads)]
                list(ex.map(lambda ab: oracle.linear_rows(c, sc, cb, k, xr, m, ab[0], ab[1]) if ab[1] > ab[0]
                            else None, chunks))
                t = time.perf_counter() - ts
                t_phase_full += t * n / r
                t_all += t
                done += r
            t_all += t_rht
            t_full += t_phase_full
    return t_all, t_full, done


def oracle_sample_frac(shape, m, budget_s, threads):
    """Fraction of each op's rows whose oracle run takes about budget_s on
    `threads` threads (from a 2-row probe of every op, single-threaded)."""
    import oracle
    oracle.build()
    _, t_layer_1, _ = oracle_layer_sample(shape, m, 0.0, 1)  # 1 row of each op -> full-layer estimate
    t_layer_par = t_layer_1 / max(1, threads)
    return min(1.0, budget_s / max(t_layer_par, 1e-9))


def oracle_baseline(shape, m, budget_s=8.0):
    """The oracle timed on the host's cores: the same sample run on all host
    cores and on one; tokens/s of the whole stack extrapolated from it."""
    cores = host_cores()
    frac = oracle_sample_frac(shape, m, budget_s, cores)
    t_par, full_par, rows = oracle_layer_sample(shape, m, frac, cores)
    t_one, full_one, _ = oracle_layer_sample(shape, m, frac, 1)
    full_rows = sum(n for _, n, _ in shape.ops())
    sample = (f"{rows} of the {full_rows} weight rows of layer 0 (the same fraction of each of its 7 ops, "
              f"with the 4 RHTs of that layer's phase seeds), m={m}; each op's time scaled by its row count, then "
              f"to {shape.layers} layers; {t_par:.1f} s on {cores} threads, {t_one:.1f} s on 1")
    return {"value": m / (full_par * shape.layers), "unit": "tok/s", "cores": cores, "kind": "oracle",
            "sample": sample, "single_thread_value": m / (full_one * shape.layers), "host_cores": cores}


def run_reference(args, shape, m):
    import oracle
    oracle.build()
    steps, warm = args.steps, args.warmup
    cores = host_cores()
    # per-step CPU budget so that warmup + steps end in about two minutes
    budget = max(2.0, 120.0 / max(1, steps + warm))
    frac = oracle_sample_frac(shape, m, budget, cores)
    for _ in range(warm):
        oracle_layer_sample(shape, m, frac, cores)
    runs = [oracle_layer_sample(shape, m, frac, cores) for _ in range(steps)]
    t_step = float(np.mean([r[0] for r in runs]))
    t_token = float(np.mean([r[1] for r in runs])) * shape.layers / m
    value = 1.0 / t_token
    full_rows = sum(n for _, n, _ in shape.ops())
    sample = (f"{runs[0][2]} of the {full_rows} weight rows of layer 0 (the same fraction of each of its 7 ops, "
              f"with the 4 RHTs of that layer's phase seeds) at m={m} per step on {cores} threads, scaled by rows "
              f"and by {shape.layers} layers")
    cpu = {"value": value, "unit": "tok/s", "cores": cores, "kind": "oracle", "sample": sample}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": warm, "ms_per_step": t_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{shape.name} stack, {shape.layers} layers, batch {m}", "layers": shape.layers,
                       "batch": m, "parallelism": "replicas"},
            "cpu_baseline": cpu, "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0,
                                         "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---- the batch-1 decode-GEMV on its own (first half of the metric) --------------------

GEMV_SHAPE = (32768, 16384)  # 138 MB packed: larger than the 126 MB L2 on its own
GEMV_COPIES = 2              # distinct weights read in turn: 277 MB per round


def bench_gemv(tq, dev, stream, steps, warmup, hbm):
    """tq_gemv on GEMV_COPIES distinct n x k weights in turn, launches replayed
    from a CUDA graph; each launch reads a weight the previous launch did not
    touch, and the copies together are twice the L2, so no launch starts with
    its weight in L2.  Returns the JSON object (GB/s over algorithmic bytes)."""
    import torch
    n, k = GEMV_SHAPE
    ws = []
    for c in range(GEMV_COPIES):
        ws.append(tq.DeviceWeight.from_host(tqsynth.codes(0, 100 + c, 0, n, k), tqsynth.scales(0, 100 + c, 0, n, k),
                                            tqsynth.codebook(0), n, k, device=dev))
    x = torch.from_numpy(tqsynth.bf16_to_f64(tqsynth.activations(0, 1, k))[0].astype(np.float32)).to(dev)
    y = torch.empty(n, dtype=torch.float32, device=dev)
    wsp = tq.workspace(tq.tq_gemv_workspace(n, k), dev)
    per_graph = 2 * GEMV_COPIES
    with torch.cuda.stream(stream):
        for i in range(per_graph):
            tq.tq_gemv(ws[i % GEMV_COPIES], x, y, wsp, stream=stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(per_graph):
            tq.tq_gemv(ws[i % GEMV_COPIES], x, y, wsp, stream=stream)
    reps = max(3, steps)
    for _ in range(max(3, warmup)):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        time.sleep(0.3)
        t0 = time.perf_counter()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        stream.synchronize()
        clk.mark(t0, time.perf_counter())
    us = e0.elapsed_time(e1) * 1e3 / (reps * per_graph)
    packed = tqsynth.pack_bytes(n, k)
    alg = packed + 16384 + 4 * k + 4 * n  # codes + scales, codebook, x' fp32, y fp32
    gbs = alg / (us * 1e-6) / 1e9
    return {"workload": f"one {n} x {k} trellis-coded weight ({packed / 1e6:.1f} MB packed), batch 1, "
                        f"{GEMV_COPIES} distinct copies read in turn ({GEMV_COPIES * packed / 1e6:.0f} MB > 126 MB L2)",
            "kernel": "dmma_kernel<LV=3, hilo> (tq_gemv: register decode + mma.sync)",
            "us_per_launch": us, "launches": reps * per_graph, "compressed_weight_gbs": packed / (us * 1e-6) / 1e9,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "bytes_per_launch": alg},
            "clocks": clk.summary()}


# ---- our arm ------------------------------------------------------------------------

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
    ap.add_argument("--no-gemv", action="store_true", help="skip the stand-alone decode-GEMV measurement")
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

    # the decode-GEMV on its own (every rank runs it on its own GPU; rank 0 reports)
    gemv = None if args.no_gemv else bench_gemv(tq, dev, stream, args.steps, args.warmup, measured_peaks()[0])

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(shape, m)

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
                      "phase_ms": ph_ms, "phase_bytes": pb} if m <= REGISTER_DECODE_MAX_M else
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
        "gemv": gemv,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
