"""Parity of the CUDA trellis encoder (tq_encode, through the C ABI) with the
oracle's binary32-decision encoder.

Both sides take every decision in binary32 in the same order, so codes,
scales and the per-block squared error must match bit for bit.  Inputs are
seeded (tqsynth); rotated inputs are rotated by the oracle and rounded to
fp32, then handed to both sides.  Nothing on the oracle side comes from the
CUDA path.
"""
import math

import numpy as np
import pytest

import oracle
import tqsynth
from gpu_util import f32_exact, to_dev_u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available()
    return torch


@pytest.fixture(scope="module")
def tq():
    import decode_matmul_b200 as m
    return m


def _gain(cb_bits):
    return float(np.float32(1.0 / math.sqrt(float((tqsynth.f16_to_f64(cb_bits) ** 2).mean()))))


def _gpu_encode(tq, torch, w32, cb_bits, gain, refits):
    w_d = torch.from_numpy(np.ascontiguousarray(w32, dtype=np.float32)).cuda()
    codes, scales, err = tq.tq_encode(w_d, to_dev_u16(cb_bits.reshape(-1)), gain, refits)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy().view(np.uint16), err.cpu().numpy()


def _assert_same(got, want):
    gc, gs, ge = got
    wc, ws, we = want
    assert np.array_equal(gs, ws), np.argwhere(gs != ws)[:5]
    assert np.array_equal(gc, wc), np.argwhere(gc != wc)[:5]
    assert np.array_equal(ge.view(np.uint32), we.view(np.uint32))


@pytest.mark.parametrize("n,k,refits", [(37, 1024, 0), (37, 1024, 1), (6, 2560, 2), (1, 512, 4)])
def test_encode_bit_exact_gaussian(tq, torch_cuda, n, k, refits):
    cb = tqsynth.codebook(3)
    w = tqsynth.weight_rows_f32(7, n, k)
    g = _gain(cb)
    _assert_same(_gpu_encode(tq, torch_cuda, w, cb, g, refits), oracle.encode32(w, cb, g, refits))


def test_encode_bit_exact_rotated_outlier_rows(tq, torch_cuda):
    # unquantized bf16 rows with outliers, rotated by the oracle (fp64 -> fp32)
    n, k = 9, 1536
    wb = tqsynth.dense_weights(11, n, k, outlier_rate=1 / 256)
    w = f32_exact(oracle.rht(wb, n, k, 0x5EED)).astype(np.float32)
    cb = tqsynth.codebook(4)
    g = _gain(cb)
    _assert_same(_gpu_encode(tq, torch_cuda, w, cb, g, 1), oracle.encode32(w, cb, g, 1))


def test_encode_edge_blocks(tq, torch_cuda):
    # zero block, constant-magnitude block, a tiny block (subnormal fp16 scale),
    # a wide-range block, and a gain that does not match the codebook
    k = 512
    rng = np.random.default_rng(1)
    rows = [np.zeros(k), 3.0 * rng.choice([-1.0, 1.0], size=k), rng.standard_normal(k) * 1e-7,
            rng.standard_normal(k) * 30.0, np.concatenate([np.zeros(256), rng.standard_normal(256)])]
    w = np.stack(rows).astype(np.float32)
    cb = tqsynth.codebook(5)
    for gain, refits in [(_gain(cb), 2), (0.37, 1), (4.0, 0)]:
        _assert_same(_gpu_encode(tq, torch_cuda, w, cb, gain, refits), oracle.encode32(w, cb, gain, refits))


def test_encode_decodes_through_the_library(tq, torch_cuda):
    # the encoder's output is a valid weight: tq_decode of it equals the oracle
    # decode of the oracle's encoding, and its error is the reported err
    n, k = 16, 1024
    cb = tqsynth.codebook(6)
    w = tqsynth.weight_rows_f32(8, n, k)
    g = _gain(cb)
    codes, scales, err = _gpu_encode(tq, torch_cuda, w, cb, g, 1)
    dw = tq.DeviceWeight.from_host(codes, scales, cb, n, k)
    got = tq.tq_decode(dw).cpu().numpy().view(np.uint16)
    wc, ws, _ = oracle.encode32(w, cb, g, 1)
    assert np.array_equal(got, oracle.decode(wc, ws, cb, n, k))
    wh = got.view(np.float16).astype(np.float64)
    sq = ((w.astype(np.float64) - wh) ** 2).reshape(n, k // 256, 256).sum(axis=2)
    assert np.allclose(err, sq, rtol=1e-5, atol=0)


def test_encode_rotation_pipeline_on_the_gpu(tq, torch_cuda):
    # tq_rht of the weight rows (the rotation the matmul applies to the
    # activations), then tq_encode: the rotated input matches the oracle's
    # rotation within the RHT tolerance and the encoding's MSE sits between the
    # distortion-rate bound and the best 2-bit scalar quantizer (relative to the
    # rows' variance)
    n, k = 64, 2048
    wb = tqsynth.dense_weights(12, n, k)
    wr = tq.tq_rht(to_dev_u16(wb), 0xABCD)
    ref = oracle.rht(wb, n, k, 0xABCD)
    got = wr.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got - ref)) <= 1e-5 * np.max(np.abs(ref))
    cb = tqsynth.codebook(0)
    codes, scales, err = tq.tq_encode(wr, to_dev_u16(cb.reshape(-1)), _gain(cb), 1)
    torch_cuda.cuda.synchronize()
    mse = float(err.double().sum().item()) / (n * k)
    var = float((ref ** 2).mean())
    assert 2.0 ** (-2 * 2.0625) < mse / var < 0.1175


def test_encode_full_size_sampled_rows(tq, torch_cuda):
    # a 4096 x 4096 matrix encoded in one launch; sampled rows bit-exact
    n, k = 4096, 4096
    cb = tqsynth.codebook(0)
    g = _gain(cb)
    w = tqsynth.weight_rows_f32(9, n, k)
    codes, scales, err = _gpu_encode(tq, torch_cuda, w, cb, g, 1)
    for r in (0, 1, 2047, 3001, 4095):
        wc, ws, we = oracle.encode32(w[r:r + 1], cb, g, 1)
        _assert_same((codes[r:r + 1], scales[r:r + 1], err[r:r + 1]), (wc, ws, we))


# ---- block LDLQ ------------------------------------------------------------------------------

def _gpu_ldlq(tq, torch, w32, u32, cb_bits, gain, refits):
    w_d = torch.from_numpy(np.ascontiguousarray(w32, dtype=np.float32)).cuda()
    u_d = torch.from_numpy(np.ascontiguousarray(u32, dtype=np.float32)).cuda()
    codes, scales, err = tq.tq_ldlq_encode(w_d, u_d, to_dev_u16(cb_bits.reshape(-1)), gain, refits)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy().view(np.uint16), err.cpu().numpy()


@pytest.mark.parametrize("n,k,gamma,refits", [(37, 1024, 0.5, 1), (70, 1536, 2.0, 0), (1, 512, 1.0, 2)])
def test_ldlq_bit_exact(tq, torch_cuda, n, k, gamma, refits):
    cb = tqsynth.codebook(13)
    w = tqsynth.weight_rows_f32(14, n, k)
    u = tqsynth.hessian_factor(15, k, gamma)
    g = _gain(cb)
    _assert_same(_gpu_ldlq(tq, torch_cuda, w, u, cb, g, refits), oracle.ldlq32(w, u, cb, g, refits))


def test_ldlq_without_feedback_equals_encode(tq, torch_cuda):
    n, k = 20, 1024
    cb = tqsynth.codebook(16)
    w = tqsynth.weight_rows_f32(17, n, k)
    g = _gain(cb)
    _assert_same(_gpu_ldlq(tq, torch_cuda, w, np.zeros((k, k), np.float32), cb, g, 1),
                 _gpu_encode(tq, torch_cuda, w, cb, g, 1))


def test_ldlq_full_size_sampled_rows(tq, torch_cuda):
    n, k = 1024, 4096
    cb = tqsynth.codebook(0)
    g = _gain(cb)
    w = tqsynth.weight_rows_f32(18, n, k)
    u = tqsynth.hessian_factor(19, k, 0.5)
    codes, scales, err = _gpu_ldlq(tq, torch_cuda, w, u, cb, g, 1)
    for r in (0, 511, 1023):
        _assert_same((codes[r:r + 1], scales[r:r + 1], err[r:r + 1]), oracle.ldlq32(w[r:r + 1], u, cb, g, 1))



def test_encode_and_ldlq_without_error_output(tq, torch_cuda):
    # err_d = NULL: the same codes and scales, nothing else written
    import torch
    n, k = 9, 1024
    cb = tqsynth.codebook(20)
    g = _gain(cb)
    w = tqsynth.weight_rows_f32(21, n, k)
    u = tqsynth.hessian_factor(22, k, 0.5)
    w_d = torch.from_numpy(w).cuda()
    u_d = torch.from_numpy(u).cuda()
    cbd = to_dev_u16(cb.reshape(-1))
    c1, s1, e1 = tq.tq_encode(w_d, cbd, g, 1, want_err=False)
    c2, s2, e2 = tq.tq_ldlq_encode(w_d, u_d, cbd, g, 1, want_err=False)
    torch.cuda.synchronize()
    assert e1 is None and e2 is None
    wc, ws, _ = oracle.encode32(w, cb, g, 1)
    assert np.array_equal(c1.cpu().numpy(), wc) and np.array_equal(s1.cpu().numpy().view(np.uint16), ws)
    lc, ls, _ = oracle.ldlq32(w, u, cb, g, 1)
    assert np.array_equal(c2.cpu().numpy(), lc) and np.array_equal(s2.cpu().numpy().view(np.uint16), ls)


def test_ldlq_wide_feedback_tiles(tq, torch_cuda):
    # enough rows for the 64-row feedback tiles (n >= 4736 on 148 SMs); sampled rows bit-exact
    n, k = 4800, 1024
    cb = tqsynth.codebook(23)
    g = _gain(cb)
    w = tqsynth.weight_rows_f32(24, n, k)
    u = tqsynth.hessian_factor(25, k, 0.5)
    codes, scales, err = _gpu_ldlq(tq, torch_cuda, w, u, cb, g, 0)
    for r in (0, 63, 64, 2399, 4799):
        _assert_same((codes[r:r + 1], scales[r:r + 1], err[r:r + 1]), oracle.ldlq32(w[r:r + 1], u, cb, g, 0))
