"""Single-kernel cases for timing and profiling (one op, seeded inputs).

    python -m decode_matmul_b200.cases gemv --n 32768 --k 16384 [--reps 10] [--flush]
    python -m decode_matmul_b200.cases gemm --n 19456 --k 2560 --m 512 [--reps 10]
    python -m decode_matmul_b200.cases rht  --m 512 --k 9728 [--reps 10]
    python -m decode_matmul_b200.cases encode --n 4096 --k 14336 [--refits 0] [--reps 5]
    python -m decode_matmul_b200.cases ldlq --n 4096 --k 4096 [--refits 0] [--reps 3]

Runs `reps` launches after 3 warm-up launches and prints the mean time per
launch (CUDA events) with the algorithmic bytes or FLOPs per launch.  For the
encoder the work unit is one Viterbi candidate (a code from a predecessor
state for one group: 5 FP32 operations); with --refits 0 every block runs
exactly one pass of 64 groups x 2048 candidates.  The
same command line is what the ncu summaries under profiles/ were taken on.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main(argv=None):
    import torch

    import decode_matmul_b200 as tq
    import tqsynth

    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["gemv", "gemm", "rht", "encode", "ldlq"])
    ap.add_argument("--refits", type=int, default=0)
    ap.add_argument("--n", type=int, default=32768)
    ap.add_argument("--k", type=int, default=16384)
    ap.add_argument("--m", type=int, default=1)
    ap.add_argument("--reps", type=int, default=10)
    ap.add_argument("--flush", action="store_true",
                    help="time each launch alone, after writing 256 MB (twice the L2) between launches")
    ap.add_argument("--graph", action="store_true",
                    help="time launches replayed from a CUDA graph (no host launch cost); with --flush, a "
                         "graph of (256 MB write + launch) minus a graph of the writes alone")
    a = ap.parse_args(argv)
    dev = torch.device("cuda", 0)

    if a.op == "ldlq":
        g = torch.Generator(device=dev)
        g.manual_seed(0)
        w = torch.randn((a.n, a.k), device=dev, generator=g)
        u = torch.from_numpy(tqsynth.hessian_factor(0, a.k, 0.5)).to(dev)
        cbh = tqsynth.codebook(0)
        cb = torch.from_numpy(cbh.reshape(-1).view(np.int16)).to(dev)
        gain = float(np.float32(1.0 / np.sqrt((tqsynth.f16_to_f64(cbh) ** 2).mean())))
        codes = torch.empty((a.n, a.k // 4), dtype=torch.uint8, device=dev)
        scales = torch.empty((a.n, a.k // 256), dtype=torch.int16, device=dev)
        err = torch.empty((a.n, a.k // 256), dtype=torch.float32, device=dev)
        ws = torch.empty(tq.tq_ldlq_workspace(a.n, a.k), dtype=torch.uint8, device=dev)
        run = lambda: tq.tq_ldlq_encode(w, u, cb, gain, a.refits, codes, scales, err, ws=ws)  # noqa: E731
        kb = a.k // 256
        work, unit = 2.0 * a.n * 256 * 256 * kb * (kb - 1) / 2, "FLOP(feedback)"
    elif a.op == "encode":
        g = torch.Generator(device=dev)
        g.manual_seed(0)
        w = torch.randn((a.n, a.k), device=dev, generator=g)
        cbh = tqsynth.codebook(0)
        cb = torch.from_numpy(cbh.reshape(-1).view(np.int16)).to(dev)
        gain = float(np.float32(1.0 / np.sqrt((tqsynth.f16_to_f64(cbh) ** 2).mean())))
        codes = torch.empty((a.n, a.k // 4), dtype=torch.uint8, device=dev)
        scales = torch.empty((a.n, a.k // 256), dtype=torch.int16, device=dev)
        err = torch.empty((a.n, a.k // 256), dtype=torch.float32, device=dev)
        run = lambda: tq.tq_encode(w, cb, gain, a.refits, codes, scales, err)  # noqa: E731
        work, unit = a.n * (a.k // 256) * 64.0 * 2048, "cand"
    elif a.op == "rht":
        x = torch.from_numpy(tqsynth.activations(0, a.m, a.k).view(np.int16)).to(dev)
        out = torch.empty((a.m, a.k), dtype=torch.float16, device=dev)
        run = lambda: tq.tq_rht(x, 1, tq.TQ_F16, out=out)  # noqa: E731
        work, unit = a.m * a.k * 4, "B"
    else:
        w = tqsynth.Weight(0, 0, 0, a.n, a.k)
        dw = tq.DeviceWeight.from_host(w.codes, w.scales, w.codebook, a.n, a.k, device=dev)
        if a.op == "gemv":
            x = torch.randn(a.k, device=dev)
            y = torch.empty(a.n, device=dev)
            ws = tq.workspace(tq.tq_gemv_workspace(a.n, a.k), dev)
            run = lambda: tq.tq_gemv(dw, x, y, ws)  # noqa: E731
            work, unit = tqsynth.pack_bytes(a.n, a.k) + 16384 + 4 * a.k + 4 * a.n, "B"
        else:
            x = torch.randn((a.m, a.k), device=dev).half()
            y = torch.empty((a.m, a.n), device=dev)
            ws = tq.workspace(tq.tq_gemm_workspace(a.n, a.k, a.m), dev)
            run = lambda: tq.tq_gemm(dw, x, y, ws)  # noqa: E731
            work, unit = 2.0 * a.m * a.n * a.k, "FLOP"
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if a.graph:
        scrub = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if a.flush else None

        def graph_ms(with_run):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(a.reps):
                    if scrub is not None:
                        scrub.fill_(i & 0xFF)
                    if with_run:
                        run()
            g.replay()
            torch.cuda.synchronize()
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / a.reps

        ms = graph_ms(True) - (graph_ms(False) if a.flush else 0.0)
    elif a.flush:
        # each launch timed on its own (median), after the L2 has been overwritten
        scrub = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        times = []
        for i in range(a.reps):
            scrub.fill_(i & 0xFF)
            e0.record()
            run()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        ms = float(np.median(times))
    else:
        e0.record()
        for _ in range(a.reps):
            run()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / a.reps
    rate = work / (ms * 1e-3)
    how = (" (graph" + (", L2 flushed" if a.flush else "") + ")") if a.graph else (" (L2 flushed, median)" if a.flush else "")
    print(f"{a.op} n={a.n} k={a.k} m={a.m}{how}: {ms * 1e3:.2f} us/launch, "
          f"{rate / 1e9:.1f} G{unit}/s ({work:.4g} {unit} per launch)")
    if a.op == "ldlq":
        # the same matrix without feedback, to split the time, and the proxy loss
        # |E (I + U)|^2 of both encodings (H = (I + U)(I + U)^T)
        c0 = torch.empty_like(codes)
        s0 = torch.empty_like(scales)
        e0 = torch.empty_like(err)
        tq.tq_encode(w, cb, gain, a.refits, c0, s0, e0)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(a.reps):
            tq.tq_encode(w, cb, gain, a.refits, c0, s0, e0)
        t1.record()
        torch.cuda.synchronize()
        ms_enc = t0.elapsed_time(t1) / a.reps
        ud = u.double() + torch.eye(a.k, device=dev, dtype=torch.float64)
        losses = []
        for cc, ss in ((codes, scales), (c0, s0)):
            wh = tq.tq_decode(tq.DeviceWeight(cc, ss, cb, a.n, a.k)).view(torch.float16).double()
            losses.append(float(((w.double() - wh) @ ud).pow(2).sum().item()))
        ms_fb = ms - ms_enc
        peak = torch.cuda.get_device_properties(0).multi_processor_count * 128 * 2 * 1.965e9
        print(f"  plain encode {ms_enc * 1e3:.1f} us; feedback + step overhead {ms_fb * 1e3:.1f} us = "
              f"{work / (ms_fb * 1e-3) / 1e12:.2f} TFLOP/s ({work / (ms_fb * 1e-3) / peak:.3f} of the FP32 peak "
              f"{peak / 1e12:.1f} TFLOP/s); proxy loss LDLQ / plain = {losses[0] / losses[1]:.4f}")
    if a.op == "encode":
        # independent 2-bit rounding at equal bytes (2 bits per weight + one
        # fp16 scale per 256 weights), on the same rows, for comparison: four
        # levels per block, nearest level for every weight on its own
        blk = w.view(-1, 256).double()
        rms = blk.pow(2).mean(dim=1, keepdim=True).sqrt()

        def scalar_mse(levels):  # levels in units of the block's fp16-rounded scale
            sc = rms.half().double()
            lv = torch.tensor(levels, dtype=torch.float64, device=dev) * sc
            q = lv.gather(1, (blk[:, :, None] - lv[:, None, :]).abs().argmin(dim=2))
            return float((blk - q).pow(2).mean().item())

        mse_uniform = scalar_mse([-1.4936, -0.4979, 0.4979, 1.4936])  # MSE-optimal uniform step for N(0,1)
        mse_lloyd = scalar_mse([-1.5104, -0.4528, 0.4528, 1.5104])    # Lloyd-Max levels for N(0,1)
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        peak = sms * 128 * 1.965e9 / 5.0  # candidates/s at 5 FP32 operations each, 1965 MHz
        mse = float(err.double().sum().item()) / (a.n * a.k)
        print(f"  {a.n * a.k / (ms * 1e-3) / 1e9:.2f} G weights/s; candidate rate {rate / peak:.3f} of the "
              f"FP32 bound ({peak / 1e12:.2f} T cand/s); refits={a.refits}; MSE/var {mse:.5f}")
        print(f"  independent 2-bit rounding, same rows and bytes: uniform levels MSE/var {mse_uniform:.5f}, "
              f"Lloyd-Max levels {mse_lloyd:.5f}; distortion-rate bound {2 ** (-2 * 2.0625):.4f}")


if __name__ == "__main__":
    main()
