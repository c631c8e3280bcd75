"""Full-size parity of the layer stack, in the launch configuration the
benchmark times, on sampled outputs.

After tq_layer_stack returns, its workspace holds the last layer's phase
inputs and handoffs (tq_layer_stack_buffers).  Each phase of that layer is
recomputed by the oracle from the GPU's own input of that phase (teacher
forcing) on sampled rows (first, last and seeded random rows of every
handoff op) and, for large batches, sampled tokens.  Checks: handoff values
within one bf16 step plus the 2e-3 output tolerance of the oracle; the last
phase's fp32 y within 2e-3; its bf16 rounding decided exactly as the GPU
decides it (fp32 alpha times the GPU's own fp32 y).
"""
import numpy as np
import pytest

import oracle
import tqsynth
from gpu_util import TOL

pytestmark = pytest.mark.gpu

# (stack, layers, batch): the Qwen3-4B-shaped stack at batch 1 runs all 36
# layers as the benchmark does; the others run two full-size layers (every
# phase is its own launch or its own phase of the persistent kernel, so the
# per-phase launch configuration is the benchmark's).
CASES = [("qwen3-4b-shaped", 36, 1), ("qwen3-4b-shaped", 2, 512),
         ("llama-3.1-8b-shaped", 2, 1), ("llama-3.1-8b-shaped", 2, 4), ("llama-3.1-8b-shaped", 2, 8),
         ("llama-3.1-8b-shaped", 2, 16),
         ("27b-class", 2, 1), ("27b-class", 2, 8), ("27b-class", 2, 32), ("27b-class", 2, 64)]


def _rows(n, rng):
    r = rng.integers(8, n - 16)
    return [(0, 8), (int(r), int(r) + 8), (n - 8, n)]


@pytest.mark.parametrize("stack,layers,m", CASES)
def test_stack_last_layer_teacher_forced(stack, layers, m):
    import torch

    import decode_matmul_b200 as tq
    seed = 0
    shape = tqsynth.stack_shape(stack, layers)
    dev = torch.device("cuda", 0)
    cb = tqsynth.codebook(seed)
    cbd = torch.from_numpy(cb.view(np.int16)).to(dev)
    host_last = {}
    dlayers = []
    for l in range(layers):
        w = {}
        for i, (op, n, k) in enumerate(shape.ops()):
            c, s = tqsynth.codes(seed, l, i, n, k), tqsynth.scales(seed, l, i, n, k)
            if l == layers - 1:
                host_last[op] = (c, s, cb, n, k)
            w[op] = tq.DeviceWeight.from_host(c, s, cbd, n, k, device=dev)
        dlayers.append(w)
    structs = [tq.layer_struct(w) for w in dlayers]
    h_in = tqsynth.activations(seed, m, shape.hidden)
    h_in_d = torch.from_numpy(h_in.view(np.int16)).to(dev)
    h_out = torch.empty_like(h_in_d)
    ws = tq.workspace(tq.tq_layer_stack_workspace(structs, m), dev)
    tq.tq_layer_stack(tq.StackArgs(structs, m), h_in_d, seed, h_out, ws)
    torch.cuda.synchronize()
    off = tq.tq_layer_stack_buffers(structs, m)
    wsn = ws.cpu().numpy()

    def buf(o, rows, cols, dt=np.uint16):
        nb = rows * cols * np.dtype(dt).itemsize
        return wsn[o:o + nb].view(dt).reshape(rows, cols)

    l = layers - 1
    ins = [h_in if layers == 1 else buf(off[3], m, shape.hidden), buf(off[0], m, shape.q_dim),
           buf(off[1], m, shape.hidden), buf(off[2], m, shape.inter)]
    outs = [buf(off[0], m, shape.q_dim), buf(off[1], m, shape.hidden), buf(off[2], m, shape.inter),
            h_out.cpu().numpy().view(np.uint16)]
    y_last = buf(off[4], m, shape.hidden, np.float32)
    rng = np.random.default_rng(1234 + m)
    toks = np.arange(m) if m <= 16 else np.unique(np.concatenate([np.arange(4), np.arange(m - 4, m),
                                                                  rng.integers(0, m, 8)]))
    for p in range(4):
        hop = oracle.HANDOFF_OP[p]
        c, s, cbh, n, k = host_last[hop]
        x = np.ascontiguousarray(ins[p][toks])
        xr = oracle.rht(x, len(toks), k, oracle.stack_phase_seed(seed, l, p))
        alpha = oracle.alpha(k)
        for r0, r1 in _rows(n, rng):
            want_y = oracle.linear_rows(c, s, cbh, k, xr, len(toks), r0, r1)
            got_h = tqsynth.bf16_to_f64(outs[p][toks, r0:r1])
            want_h = tqsynth.bf16_to_f64(oracle.handoff(want_y, k))
            rms = np.sqrt(np.mean(want_h * want_h))
            bound = np.abs(want_h) * 2.0 ** -7 + TOL * np.maximum(np.abs(want_h), rms)
            assert np.all(np.abs(got_h - want_h) <= bound), (p, r0)
            if p == 3:
                yg = y_last[toks, r0:r1]
                assert oracle.rel_err(yg, want_y) < TOL, (r0, oracle.rel_err(yg, want_y))
                a32 = np.float32(alpha)
                expect = oracle.bf16_from_f64((a32 * yg.astype(np.float32)).astype(np.float64))
                assert np.array_equal(outs[p][toks, r0:r1], expect)
