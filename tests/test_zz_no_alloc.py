"""tq_gemv_noalloc: batch-1 GEMV for callers that cannot give the library any
device memory (a runtime that owns every allocation and offers no workspace
hook, or a path that must not call cudaMalloc).  Its scratch is a fixed
device array inside the library.  This file is collected last on purpose.

The test calls the entry point through the C ABI twice in a row (the second
call finds the array as the first left it) and compares each result with the
workspace-taking tq_gemv; it also checks the size limit is refused."""
import ctypes

import numpy as np
import pytest

import oracle
import tqsynth
from gpu_util import TOL, dev_weight, host_weight


@pytest.mark.gpu
def test_gemv_noalloc_matches_gemv_on_two_calls():
    import torch

    import decode_matmul_b200 as tq
    L = tq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # beyond the built-in scratch: refused before anything is launched
    big = tq.tq_weight_t(16, 16, 16, 262160, 512)
    assert L.tq_gemv_noalloc(ctypes.byref(big), 16, 16, stream) == tq.TQ_ERR_SCRATCH
    for n, k in [(1024, 1024), (2560, 9728), (37, 512)]:
        hw = host_weight(7, 0, 3, n, k)
        w = dev_weight(hw)
        x = torch.from_numpy(tqsynth.bf16_to_f64(tqsynth.activations(3, 1, k))[0].astype(np.float32)).cuda()
        ref = tq.tq_gemv(w, x)
        torch.cuda.synchronize()
        ws = w.struct()
        for _ in range(2):
            y = torch.full((n,), float("nan"), device="cuda")
            st = L.tq_gemv_noalloc(ctypes.byref(ws), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()),
                                   stream)
            assert st == tq.TQ_OK, tq.lib().tq_status_string(st)
            torch.cuda.synchronize()
            assert oracle.rel_err(y.cpu().numpy(), ref.cpu().numpy()) < TOL
