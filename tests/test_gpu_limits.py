"""The CUDA path at the documented size limits, against the oracle on sampled
outputs: the most rows a decode-GEMV call takes (262128 = 16383 tiles of 16),
the widest input it takes (TQ_GEMV_MAX_K = 53760 features) and the most
tokens a GEMM call takes (4096); one past each is rejected."""
import ctypes

import numpy as np
import pytest

import oracle
import tqsynth
from gpu_util import TOL, dev_weight, f16_exact, f32_exact, host_weight

pytestmark = pytest.mark.gpu


def test_gemv_at_the_row_limit():
    import torch

    import decode_matmul_b200 as tq
    n, k = 262128, 512
    hw = host_weight(3, 0, 1, n, k)
    x = tqsynth.activations(3, 1, k)
    xr = f32_exact(oracle.rht(x, 1, k, 21))
    dw = dev_weight(hw)
    y = tq.tq_gemv(dw, torch.from_numpy(xr.astype(np.float32)).cuda()).cpu().numpy()
    for r0, r1 in [(0, 16), (131064, 131080), (n - 16, n)]:
        want = oracle.linear_rows(hw.codes, hw.scales, hw.codebook, k, xr, 1, r0, r1)[0]
        assert oracle.rel_err(y[r0:r1], want) < TOL, r0
    # one row more does not fit the per-tile counters
    big = tq.tq_weight_t(dw.codes.data_ptr(), dw.scales.data_ptr(), dw.codebook.data_ptr(), n + 1, k)
    ws = tq.workspace(tq.tq_gemv_workspace(n + 1, k))
    yb = torch.empty(n + 1, dtype=torch.float32, device="cuda")
    st = tq.lib().tq_gemv(ctypes.byref(big), ctypes.c_void_p(0), ctypes.c_void_p(yb.data_ptr()),
                          ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
    assert st in (tq.TQ_ERR_SHAPE, tq.TQ_ERR_NULL)
    xd = torch.from_numpy(xr.astype(np.float32)).cuda()
    st = tq.lib().tq_gemv(ctypes.byref(big), ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(yb.data_ptr()),
                          ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
    assert st == tq.TQ_ERR_SHAPE


def test_gemm_at_the_token_limit():
    import torch

    import decode_matmul_b200 as tq
    n, k, m = 256, 512, 4096
    hw = host_weight(4, 0, 2, n, k)
    x = tqsynth.activations(4, m, k)
    xr = f16_exact(oracle.rht(x, m, k, 22))
    xd = torch.from_numpy(xr.astype(np.float16)).cuda()
    y = tq.tq_gemm(dev_weight(hw), xd).cpu().numpy()
    toks = np.array([0, 1, 2047, 2048, 4094, 4095])
    want = oracle.linear(hw.codes, hw.scales, hw.codebook, n, k, np.ascontiguousarray(xr[toks]), len(toks))
    assert oracle.rel_err(y[toks], want) < TOL
    with pytest.raises(tq.TqError) as e:
        tq.tq_gemm_workspace(n, k, m + 1)
    assert e.value.status == tq.TQ_ERR_SHAPE


def test_gemv_at_the_k_limit():
    import torch

    import decode_matmul_b200 as tq
    n, k = 40, tq.TQ_GEMV_MAX_K
    hw = host_weight(5, 0, 4, n, k)
    x = tqsynth.activations(5, 1, k)
    xr = f32_exact(oracle.rht(x, 1, k, 23))
    dw = dev_weight(hw)
    xd = torch.from_numpy(xr.astype(np.float32)).cuda()
    y = tq.tq_gemv(dw, xd).cpu().numpy()
    want = oracle.linear(hw.codes, hw.scales, hw.codebook, n, k, xr, 1)[0]
    assert oracle.rel_err(y, want) < 1e-4
    # one 512-block wider does not fit shared memory: refused, nothing launched
    wide = tq.tq_weight_t(dw.codes.data_ptr(), dw.scales.data_ptr(), dw.codebook.data_ptr(), n, k + 512)
    ws = tq.workspace(tq.tq_gemv_workspace(n, k + 512))
    yb = torch.empty(n, dtype=torch.float32, device="cuda")
    st = tq.lib().tq_gemv(ctypes.byref(wide), ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(yb.data_ptr()),
                          ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
    assert st == tq.TQ_ERR_SHAPE
