"""Single-kernel cases for timing and profiling (one op, seeded inputs).

    python -m decode_matmul_b200.cases gemv --n 32768 --k 16384 [--reps 10]
    python -m decode_matmul_b200.cases gemm --n 19456 --k 2560 --m 512 [--reps 10]
    python -m decode_matmul_b200.cases rht  --m 512 --k 9728 [--reps 10]

Runs `reps` launches after 3 warm-up launches and prints the mean time per
launch (CUDA events) with the algorithmic bytes or FLOPs per launch.  The
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
    ap.add_argument("op", choices=["gemv", "gemm", "rht"])
    ap.add_argument("--n", type=int, default=32768)
    ap.add_argument("--k", type=int, default=16384)
    ap.add_argument("--m", type=int, default=1)
    ap.add_argument("--reps", type=int, default=10)
    a = ap.parse_args(argv)
    dev = torch.device("cuda", 0)

    if a.op == "rht":
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
    e0.record()
    for _ in range(a.reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.reps
    rate = work / (ms * 1e-3)
    print(f"{a.op} n={a.n} k={a.k} m={a.m}: {ms * 1e3:.2f} us/launch, "
          f"{rate / 1e9:.1f} G{unit}/s ({work:.4g} {unit} per launch)")


if __name__ == "__main__":
    main()
