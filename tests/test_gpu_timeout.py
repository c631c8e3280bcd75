"""The timeout paths, made to happen on purpose by host-side test hooks:
- the persistent stack kernels: one thread block skips its arrive at the
  launch's first grid barrier (tq_layer_stack_ex), so every block's bounded
  wait runs out after a short poll limit;
- the tcgen05 GEMM (tq_gemm_ex at 33 tokens and more): one thread block's
  decoded-stage barriers expect one arrival more than its decoders make, so
  its MMA thread's bounded wait runs out and the block drains its copies.
Each launch must end by itself, leave TQ_ERR_TIMEOUT in the workspace's
status word, and leave the context usable: after tq_workspace_init the same
workspace gives the same bits as a clean run.  Nothing here faults the GPU:
every wait in those kernels is bounded."""
import ctypes

import numpy as np
import pytest

import tqsynth

pytestmark = pytest.mark.gpu


def _small_stack(tq, dev, layers=2):
    shape = tqsynth.StackShape("timeout-test", layers, 512, 1024, 512, 1536)
    cb = tqsynth.codebook(9)
    import torch
    cbd = torch.from_numpy(cb.view(np.int16)).to(dev)
    structs, keep = [], []
    for l in range(layers):
        w = {}
        for i, (op, n, k) in enumerate(shape.ops()):
            w[op] = tq.DeviceWeight.from_host(tqsynth.codes(9, l, i, n, k), tqsynth.scales(9, l, i, n, k), cbd, n, k,
                                              device=dev)
        keep.append(w)
        structs.append(tq.layer_struct(w))
    return shape, structs, keep


@pytest.mark.parametrize("m", [1, 4])
def test_stack_wait_runs_out_then_the_workspace_recovers(m):
    import torch

    import decode_matmul_b200 as tq
    dev = torch.device("cuda", 0)
    shape, structs, _keep = _small_stack(tq, dev)
    args = tq.StackArgs(structs, m)
    nbytes = tq.tq_layer_stack_workspace(structs, m)
    h_in = torch.from_numpy(tqsynth.activations(4, m, shape.hidden).view(np.int16)).to(dev)

    ws_ref = tq.workspace(nbytes, dev)
    ref = torch.empty_like(h_in)
    tq.tq_layer_stack(args, h_in, 5, ref, ws_ref)
    assert tq.tq_workspace_status(ws_ref) == tq.TQ_OK

    ws = tq.workspace(nbytes, dev)
    out = torch.zeros_like(h_in)
    tq.tq_layer_stack_ex(args, h_in, 5, out, ws, spin_limit=2048, test_skip_arrive=3)
    assert tq.tq_workspace_status(ws) == tq.TQ_ERR_TIMEOUT

    # the context still works: a re-initialised workspace gives the clean bits
    assert tq.lib().tq_workspace_init(ctypes.c_void_p(ws.data_ptr()), ws.numel(), None) == tq.TQ_OK
    tq.tq_layer_stack(args, h_in, 5, out, ws)
    assert tq.tq_workspace_status(ws) == tq.TQ_OK
    assert torch.equal(out, ref)

    # a block index past the grid skips nothing
    out2 = torch.zeros_like(h_in)
    tq.tq_layer_stack_ex(args, h_in, 5, out2, ws, test_skip_arrive=1 << 20)
    assert tq.tq_workspace_status(ws) == tq.TQ_OK
    assert torch.equal(out2, ref)


def test_tcgen05_gemm_wait_runs_out_then_the_workspace_recovers():
    import torch

    import decode_matmul_b200 as tq
    dev = torch.device("cuda", 0)
    n, k, m = 1040, 1536, 64  # 9 row tiles, each split over k: 54 thread blocks
    hw = tqsynth.Weight(9, 0, 1, n, k)
    w = tq.DeviceWeight.from_host(hw.codes, hw.scales, hw.codebook, n, k, device=dev)
    x = torch.from_numpy(np.random.default_rng(9).standard_normal((m, k)).astype(np.float16)).to(dev)
    nbytes = tq.tq_gemm_workspace(n, k, m)

    ws_ref = tq.workspace(nbytes, dev)
    ref = tq.tq_gemm(w, x, ws=ws_ref)
    assert tq.tq_workspace_status(ws_ref) == tq.TQ_OK

    ws = tq.workspace(nbytes, dev)
    y = torch.zeros((m, n), dtype=torch.float32, device=dev)
    tq.tq_gemm_ex(w, x, y, ws, spin_limit=4096, test_skip_arrive=2)
    assert tq.tq_workspace_status(ws) == tq.TQ_ERR_TIMEOUT

    assert tq.lib().tq_workspace_init(ctypes.c_void_p(ws.data_ptr()), ws.numel(), None) == tq.TQ_OK
    y2 = torch.zeros_like(y)
    tq.tq_gemm(w, x, y2, ws)
    assert tq.tq_workspace_status(ws) == tq.TQ_OK
    assert torch.equal(y2, ref)

    # a block index past the grid skips nothing
    y3 = torch.zeros_like(y)
    tq.tq_gemm_ex(w, x, y3, ws, test_skip_arrive=1 << 20)
    assert tq.tq_workspace_status(ws) == tq.TQ_OK
    assert torch.equal(y3, ref)
