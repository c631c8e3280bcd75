"""The decode-to-shared-memory tcgen05 GEMM (tq_gemm at m >= 33) against the
oracle: tile shapes with split-k, ragged rows and several token tiles."""
import numpy as np
import pytest

import oracle
import tqsynth
from gpu_util import TOL, dev_weight, f16_exact, host_weight, oracle_linear

pytestmark = pytest.mark.gpu


def _run(n, k, m, rows=None, seed=2):
    import torch

    import decode_matmul_b200 as tq
    hw = host_weight(seed, 0, 5, n, k)
    x = tqsynth.activations(seed, m, k)
    xr = f16_exact(oracle.rht(x, m, k, 11))
    xd = torch.from_numpy(xr.astype(np.float16)).cuda()
    y = tq.tq_gemm(dev_weight(hw), xd).cpu().numpy()
    if rows is None:
        want = oracle_linear(hw, xr, m)
        return oracle.rel_err(y, want)
    errs = []
    for r0, r1 in rows:
        want = oracle.linear_rows(hw.codes, hw.scales, hw.codebook, k, xr, m, r0, r1)
        errs.append(oracle.rel_err(y[:, r0:r1], want))
    return max(errs)


@pytest.mark.parametrize("n,k,m", [(128, 512, 64), (1040, 1536, 64), (640, 2560, 128), (384, 1024, 200),
                                   (256, 512, 512)])
def test_tcgen05_gemm_full_compare(n, k, m):
    err = _run(n, k, m)
    assert err < TOL, err


def test_tcgen05_gemm_split_k_large_k():
    # 20 row tiles x 1 token tile -> split k across the blocks of k = 9728
    err = _run(2560, 9728, 64, rows=[(0, 8), (1277, 1283), (2552, 2560)])
    assert err < TOL, err


@pytest.mark.parametrize("n,k", [(19456, 2560), (14208, 1024)])
def test_tcgen05_gemm_split_tail_wave(n, k):
    # more tiles than SMs with a partial last wave (304 and 222 tiles of
    # 128 rows x 256 tokens on 148 SMs); rows sampled in the first tiles and in
    # the tiles of the last wave
    rows = [(0, 8), (5000, 5008), (n - 640, n - 632), (n - 8, n)]
    err = _run(n, k, 512, rows=rows, seed=4)
    assert err < TOL, err


@pytest.mark.parametrize("m", [40, 64, 100, 128])
def test_tcgen05_gemm_two_ctas_per_sm(m):
    # 64- and 128-token tiles with at least as many tiles as SMs run two CTAs
    # per SM
    # (149 tiles of 128 rows, the last 56 rows): every row of the first two
    # tiles, two tiles in the middle and the ragged last tile
    n = 19000
    rows = [(0, 256), (9472, 9728), (18944, n)]
    err = _run(n, 1024, m, rows=rows, seed=6)
    assert err < TOL, err


def test_tcgen05_gemm_two_ctas_per_sm_split_k():
    # 40 row tiles at 48 tokens: k = 17408 split 7 ways (about 10 blocks each)
    # for two CTAs per SM; rows of the first, a middle and the last tile
    err = _run(5120, 17408, 48, rows=[(0, 128), (2560, 2688), (4992, 5120)], seed=7)
    assert err < TOL, err
