"""tq_gemv_noalloc: batch-1 GEMV for callers that cannot give the library any
device memory (a runtime that owns every allocation and offers no workspace
hook, or a path that must not call cudaMalloc).  Its scratch is a fixed
device array inside the library.  This file is collected last on purpose.

The test calls the entry point through the C ABI twice in a row (the second
call finds the array as the first left it) and requires each result to be
bit-identical to the workspace-taking tq_gemv (the same kernel with the same
unit split and summation order) and within the tolerance of the oracle.  The
largest shape that fits the array (262128 rows at k = 512: 64 KiB of counters
plus 8192 warps' partial sums, exactly the array) runs too, checked on
sampled rows, and the first size past it is refused."""
import ctypes

import numpy as np
import pytest

import oracle
import tqsynth
from gpu_util import TOL, dev_weight, f32_exact, host_weight


def _call(tq, L, w, x, y, stream):
    ws = w.struct()
    st = L.tq_gemv_noalloc(ctypes.byref(ws), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()), stream)
    assert st == tq.TQ_OK, tq.lib().tq_status_string(st)


@pytest.mark.gpu
def test_gemv_noalloc_matches_gemv_on_two_calls():
    import torch

    import decode_matmul_b200 as tq
    L = tq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # beyond the built-in scratch: refused before anything is enqueued
    big = tq.tq_weight_t(16, 16, 16, 262160, 512)
    assert L.tq_gemv_noalloc(ctypes.byref(big), 16, 16, stream) == tq.TQ_ERR_SCRATCH
    for n, k, rows in [(1024, 1024, None), (2560, 9728, None), (37, 512, None),
                       (262128, 512, [(0, 16), (131064, 131080), (262112, 262128)])]:
        hw = host_weight(7, 0, 3, n, k)
        w = dev_weight(hw)
        xr = f32_exact(oracle.rht(tqsynth.activations(3, 1, k), 1, k, 11))
        x = torch.from_numpy(xr.astype(np.float32)).cuda()
        ref = tq.tq_gemv(w, x)
        torch.cuda.synchronize()
        for _ in range(2):
            y = torch.full((n,), float("nan"), device="cuda")
            _call(tq, L, w, x, y, stream)
            torch.cuda.synchronize()
            assert torch.equal(y, ref), (n, k)
            yh = y.cpu().numpy()
            for r0, r1 in (rows or [(0, n)]):
                want = oracle.linear_rows(hw.codes, hw.scales, hw.codebook, k, xr, 1, r0, r1)[0]
                assert oracle.rel_err(yh[r0:r1], want) < TOL, (n, k, r0)
