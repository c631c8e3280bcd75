"""Helpers for the GPU parity tests: upload seeded inputs, compare with the oracle."""
import numpy as np

import oracle
import tqsynth

TOL = 2e-3  # max relative error of an output tensor vs the fp64 oracle (fp32 accumulate)


def torch_dev():
    import torch
    return torch.device("cuda:0")


def to_dev_u16(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).to(torch_dev())


def from_dev_u16(t) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def host_weight(seed, layer, op, n, k, cb=None):
    return tqsynth.Weight(seed, layer, op, n, k, cb)


def dev_weight(hw):
    import decode_matmul_b200 as tq
    return tq.DeviceWeight.from_host(hw.codes, hw.scales, hw.codebook, hw.n, hw.k, device=torch_dev())


def oracle_linear(hw, xr, m):
    return oracle.linear(hw.codes, hw.scales, hw.codebook, hw.n, hw.k, xr, m)


def f32_exact(x64: np.ndarray) -> np.ndarray:
    """fp64 values rounded to fp32 (numpy cast, RNE) and back, as fp64."""
    return np.asarray(x64, dtype=np.float64).astype(np.float32).astype(np.float64)


def f16_exact(x64: np.ndarray) -> np.ndarray:
    return np.asarray(x64, dtype=np.float64).astype(np.float16).astype(np.float64)
