"""Parity of the CUDA path (called through the C ABI) with the oracle.

Decode must match bit for bit in fp16; GEMV / GEMM / layer-phase outputs must
be within max relative error 2e-3 of the fp64 oracle, where the error of a
tensor is max_i |y_i - ref_i| / max(|ref_i|, rms(ref)).  Inputs come from
tqsynth (seeded) or from the oracle; nothing on the oracle side comes from the
CUDA path.
"""
import numpy as np
import pytest

import oracle
import tqsynth
from gpu_util import TOL, dev_weight, f16_exact, f32_exact, from_dev_u16, host_weight, oracle_linear, to_dev_u16

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


# ---- decode ----------------------------------------------------------------------

@pytest.mark.parametrize("n,k", [(1024, 1024), (37, 512), (1, 512), (16, 2560), (100, 1536)])
def test_decode_bit_exact(tq, torch_cuda, n, k):
    hw = host_weight(0, 0, 0, n, k)
    got = from_dev_u16(tq.tq_decode(dev_weight(hw)))
    want = oracle.decode(hw.codes, hw.scales, hw.codebook, n, k)
    assert np.array_equal(got, want)



@pytest.mark.parametrize("n,k", [(2560, 9728), (4096, 14336), (5120, 17408)])
def test_decode_bit_exact_down_projection_widths(tq, torch_cuda, n, k):
    # the down projections of the three stacks (Qwen3-4B, Llama-3.1-8B and
    # 27B-class shapes), decoded whole on the GPU; sampled rows (first, last,
    # a tile boundary and 60 seeded others) against the oracle bit for bit
    hw = host_weight(0, 1, 6, n, k)
    got = from_dev_u16(tq.tq_decode(dev_weight(hw)))
    assert got.shape == (n, k)
    rows = sorted({0, 1, 15, 16, n // 2, n - 2, n - 1} | set(np.random.default_rng(k).integers(0, n, 60).tolist()))
    for r in rows:
        want = oracle.decode_rows(hw.codes, hw.scales, hw.codebook, k, r, r + 1)[0]
        assert np.array_equal(got[r], want), r

def test_decode_hand_codebook_block_reset(tq, torch_cuda):
    # the hand-worked example of tests/golden (block reset at group 64)
    s = np.arange(8)[:, None, None]
    c = np.arange(256)[None, :, None]
    j = np.arange(4)[None, None, :]
    cb = (((-1.0) ** j) * (2.0 ** (j >> 1)) * (s + c / 256.0)).astype(np.float16).view(np.uint16)
    codes = np.zeros((1, 128), dtype=np.uint8)
    codes[0, 62:66] = [14, 255, 3, 16]
    scales = np.array([[np.float16(1.0).view(np.uint16), np.float16(0.5).view(np.uint16)]], dtype=np.uint16)
    w = tq.DeviceWeight.from_host(codes, scales, cb, 1, 512)
    got = from_dev_u16(tq.tq_decode(w))
    assert np.array_equal(got, oracle.decode(codes, scales, cb, 1, 512))
    vals = got.view(np.float16).astype(np.float64).reshape(128, 4)
    assert vals[64].tolist() == [0.005859375, -0.005859375, 0.01171875, -0.01171875]


# ---- RHT ---------------------------------------------------------------------------

@pytest.mark.parametrize("m,k", [(1, 512), (3, 1536), (2, 2560)])
def test_rht_f32(tq, torch_cuda, m, k):
    x = tqsynth.activations(1, m, k)
    got = tq.tq_rht(to_dev_u16(x), 99, tq.TQ_F32).cpu().numpy().astype(np.float64)
    want = oracle.rht(x, m, k, 99)
    assert np.max(np.abs(got - want)) < 2e-5 * max(1.0, np.max(np.abs(want)))


def test_rht_f16_within_one_ulp(tq, torch_cuda):
    m, k = 4, 1024
    x = tqsynth.activations(2, m, k)
    got = tq.tq_rht(to_dev_u16(x), 5, tq.TQ_F16).cpu().numpy().astype(np.float64)
    want = oracle.rht(x, m, k, 5)
    ulp = np.spacing(np.abs(want).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(got - want) <= ulp)
    assert np.mean(got == f16_exact(want)) > 0.98


# ---- GEMV (batch 1) --------------------------------------------------------------

@pytest.mark.parametrize("n,k", [(1024, 1024), (1, 512), (17, 512), (100, 2560), (2560, 4096), (1024, 9728)])
def test_gemv(tq, torch_cuda, n, k):
    import torch
    hw = host_weight(0, 0, 0, n, k)
    x = tqsynth.activations(0, 1, k)
    xr = f32_exact(oracle.rht(x, 1, k, 7))  # the fp32 x' both sides use
    xd = torch.from_numpy(xr.astype(np.float32)).cuda()
    y = tq.tq_gemv(dev_weight(hw), xd).cpu().numpy()
    want = oracle_linear(hw, xr, 1)[0]
    err = oracle.rel_err(y, want)
    assert err < TOL, err
    assert err < 1e-4  # hi/lo split keeps the fp32 activation: expected ~1e-6


def test_gemv_deterministic_and_counters_reset(tq, torch_cuda):
    import torch
    n, k = 2560, 9728
    hw = host_weight(3, 0, 6, n, k)
    w = dev_weight(hw)
    xd = torch.randn(k, device="cuda")
    ws = tq.workspace(tq.tq_gemv_workspace(n, k))
    y1 = tq.tq_gemv(w, xd, ws=ws).clone()
    y2 = tq.tq_gemv(w, xd, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    tiles = (n + 15) // 16
    assert int(ws[: tiles * 4].view(torch.int32).abs().sum()) == 0


# ---- small-batch GEMM -------------------------------------------------------------

@pytest.mark.parametrize("m", [2, 7, 8, 16, 17, 24, 31, 32, 33, 64, 100])
def test_gemm_small_batch(tq, torch_cuda, m):
    import torch
    n, k = 1040, 1536
    hw = host_weight(1, 0, 4, n, k)
    x = tqsynth.activations(1, m, k)
    xr = f16_exact(oracle.rht(x, m, k, 3))
    xd = torch.from_numpy(xr.astype(np.float16)).cuda()
    y = tq.tq_gemm(dev_weight(hw), xd).cpu().numpy()
    want = oracle_linear(hw, xr, m)
    err = oracle.rel_err(y, want)
    assert err < TOL, err


@pytest.mark.parametrize("m", [24, 32])
def test_gemm_two_row_tiles(tq, torch_cuda, m):
    # 17-32 tokens on a shape with enough 32-row units for the two-row-tile
    # kernel (at least 5 per warp of 148 x 8): 297 tiles x 20 blocks, the last
    # tile 8 rows of 32; every tile spans about four warps, so each is summed
    # from partials.  Compared element by element on every row of the first 8
    # tiles, 8 tiles in the middle and the ragged last tile (the whole matrix
    # would take the oracle ~15 s).
    import torch
    n, k = 9480, 5120
    hw = host_weight(4, 0, 6, n, k)
    x = tqsynth.activations(4, m, k)
    xr = f16_exact(oracle.rht(x, m, k, 5))
    xd = torch.from_numpy(xr.astype(np.float16)).cuda()
    y = tq.tq_gemm(dev_weight(hw), xd).cpu().numpy()
    for r0, r1 in [(0, 256), (4736, 4992), (n - 8, n)]:
        want = oracle.linear_rows(hw.codes, hw.scales, hw.codebook, k, xr, m, r0, r1)
        err = oracle.rel_err(y[:, r0:r1], want)
        assert err < TOL, (r0, err)


@pytest.mark.parametrize("m", [32, 64])
def test_gemm_repeatable_bits(tq, torch_cuda, m):
    # tiles summed from several thread blocks' partials in a fixed order: the
    # two-row-tile kernel at 32 tokens (27B-class down projection, every tile
    # split over warps) and the tcgen05 kernel at 64 (the gate|up shape, two
    # CTAs per SM; the down projection, split k) give the same bits every call
    import torch
    for n, k in [(5120, 17408), (34816, 5120)]:
        hw = host_weight(8, 0, 2, n, k)
        w = dev_weight(hw)
        x = torch.from_numpy(np.random.default_rng(8).standard_normal((m, k)).astype(np.float16)).cuda()
        ws = tq.workspace(tq.tq_gemm_workspace(n, k, m))
        y0 = tq.tq_gemm(w, x, ws=ws)
        for _ in range(2):
            assert torch.equal(tq.tq_gemm(w, x, ws=ws), y0), (n, k, m)


# ---- layer phases ------------------------------------------------------------------

SMALL = tqsynth.StackShape("small", 2, 512, 1024, 512, 1536)


def _host_layers(shape, seed=0):
    cb = tqsynth.codebook(seed)
    layers = []
    for l in range(shape.layers):
        layers.append({op: host_weight(seed, l, i, n, k, cb) for i, (op, n, k) in enumerate(shape.ops())})
    return layers


def _dev_layers(tq, hlayers):
    # the ops of one phase must share one device codebook
    cbd = to_dev_u16(hlayers[0]["q"].codebook)
    dl = [{op: tq.DeviceWeight.from_host(hw.codes, hw.scales, cbd, hw.n, hw.k) for op, hw in L.items()}
          for L in hlayers]
    return dl, [tq.layer_struct(d) for d in dl]


def _oracle_weights(L):
    return {op: (hw.codes, hw.scales, hw.codebook, hw.n, hw.k) for op, hw in L.items()}


def _check_handoff(h_bits, y_gpu, hand_oracle, k):
    """The handoff is bf16_RNE(alpha * y) taken in fp32 on the GPU's own fp32 y
    (the rounding decision is checked in the precision it is made in); its
    value is then within one bf16 step plus the output tolerance of the
    oracle's handoff."""
    a32 = np.float32(oracle.alpha(k))
    prod = (a32 * y_gpu.astype(np.float32)).astype(np.float64)
    expect = oracle.bf16_from_f64(prod)
    assert np.mean(h_bits != expect) <= 1e-3
    got = tqsynth.bf16_to_f64(h_bits)
    want = tqsynth.bf16_to_f64(hand_oracle)
    step = np.abs(want) * 2.0 ** -7
    rms = np.sqrt(np.mean(want * want))
    assert np.all(np.abs(got - want) <= step + TOL * np.maximum(np.abs(want), rms))


@pytest.mark.parametrize("m", [1, 3, 20])
def test_layer_phases_teacher_forced(tq, torch_cuda, m):
    import torch
    hl = _host_layers(SMALL)
    dl, structs = _dev_layers(tq, hl)
    L = structs[0]
    for p in range(4):
        kin = hl[0][oracle.PHASES[p][0]].k
        n_phase = sum(hl[0][op].n for op in oracle.PHASES[p])
        n_hand = hl[0][oracle.HANDOFF_OP[p]].n
        x = tqsynth.activations(10 + p, m, kin)
        seed = tq.tq_stack_phase_seed(0, 0, p)
        y = torch.empty((m, n_phase), dtype=torch.float32, device="cuda")
        h = torch.empty((m, n_hand), dtype=torch.int16, device="cuda")
        ws = tq.workspace(tq.tq_layer_phase_workspace(L, p, m))
        tq.tq_layer_phase(L, p, to_dev_u16(x), seed, y, h, ws)
        ys, hand = oracle.stack_phase(p, x, m, _oracle_weights(hl[0]), oracle.stack_phase_seed(0, 0, p))
        want = np.concatenate([ys[op] for op in oracle.PHASES[p]], axis=1)
        err = oracle.rel_err(y.cpu().numpy(), want)
        assert err < TOL, (p, err)
        _check_handoff(from_dev_u16(h), y.cpu().numpy()[:, :n_hand], hand, hl[0][oracle.HANDOFF_OP[p]].k)


@pytest.mark.parametrize("m", [1, 3, 9, 16])
def test_layer_stack_is_the_phase_chain(tq, torch_cuda, m):
    import torch
    hl = _host_layers(SMALL)
    dl, structs = _dev_layers(tq, hl)
    x = to_dev_u16(tqsynth.activations(0, m, SMALL.hidden))
    args = tq.StackArgs(structs, m)
    ws = tq.workspace(tq.tq_layer_stack_workspace(structs, m))
    out = torch.empty_like(x)
    tq.tq_layer_stack(args, x, 42, out, ws)
    # the same chain, one phase call at a time
    cur = x
    for l, L in enumerate(structs):
        for p in range(4):
            n_phase = sum(hl[l][op].n for op in oracle.PHASES[p])
            n_hand = hl[l][oracle.HANDOFF_OP[p]].n
            y = torch.empty((m, n_phase), dtype=torch.float32, device="cuda")
            h = torch.empty((m, n_hand), dtype=torch.int16, device="cuda")
            wsp = tq.workspace(tq.tq_layer_phase_workspace(L, p, m))
            tq.tq_layer_phase(L, p, cur, tq.tq_stack_phase_seed(42, l, p), y, h, wsp)
            cur = h
    torch.cuda.synchronize()
    assert torch.equal(out, cur)
    # end-to-end drift against the oracle stack (reported, loosely bounded)
    want, _ = oracle.layer_stack([_oracle_weights(L) for L in hl], from_dev_u16(x), m, 42)
    drift = oracle.rel_err(tqsynth.bf16_to_f64(from_dev_u16(out)), tqsynth.bf16_to_f64(want))
    assert drift < 0.05, drift


# Stacks run by the persistent kernels (1-16 tokens) whose tiles straddle many
# CTAs: ragged k/v outputs (rows not a multiple of 16, never consumed), and a
# wide down projection (k = 8704 over 512 output rows: each 16-row tile spans
# about five CTAs, more than the contributors whose loads are issued together).
RAGGED = tqsynth.StackShape("ragged", 3, 1024, 1536, 200, 2560)
WIDE = tqsynth.StackShape("wide", 2, 512, 512, 96, 8704)


@pytest.mark.parametrize("m", [1, 5, 12])
@pytest.mark.parametrize("shape", [RAGGED, WIDE], ids=["ragged", "wide"])
def test_stack_persistent_straddling_tiles(tq, torch_cuda, shape, m):
    import torch
    hl = _host_layers(shape, seed=3)
    dl, structs = _dev_layers(tq, hl)
    x = to_dev_u16(tqsynth.activations(7, m, shape.hidden))
    args = tq.StackArgs(structs, m)
    ws = tq.workspace(tq.tq_layer_stack_workspace(structs, m))
    outs = []
    for _ in range(3):  # the persistent kernel is deterministic from run to run
        out = torch.empty_like(x)
        tq.tq_layer_stack(args, x, 9, out, ws)
        outs.append(out)
    torch.cuda.synchronize()
    off = tq.tq_layer_stack_buffers(structs, 1)
    y_stack = ws[off[4]:off[4] + 4 * shape.hidden].view(torch.float32).clone()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    # the last layer's outputs of every phase (ragged k / v rows included)
    yoff = tq.tq_layer_stack_outputs(structs, m)
    last = shape.layers - 1
    y_stack = []
    for p in range(4):
        n_phase = sum(hl[last][op].n for op in oracle.PHASES[p])
        y_stack.append(ws[yoff[p]:yoff[p] + 4 * m * n_phase].view(torch.float32).reshape(m, n_phase).clone())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    cur = x
    y_chain = []
    for l, L in enumerate(structs):
        for p in range(4):
            n_phase = sum(hl[l][op].n for op in oracle.PHASES[p])
            n_hand = hl[l][oracle.HANDOFF_OP[p]].n
            y = torch.empty((m, n_phase), dtype=torch.float32, device="cuda")
            h = torch.empty((m, n_hand), dtype=torch.int16, device="cuda")
            wsp = tq.workspace(tq.tq_layer_phase_workspace(L, p, m))
            tq.tq_layer_phase(L, p, cur, tq.tq_stack_phase_seed(9, l, p), y, h, wsp)
            cur = h
            if l == last:
                y_chain.append(y)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], cur)
    for p in range(4):
        assert torch.equal(y_stack[p], y_chain[p]), p
    assert tq.tq_layer_stack_buffers(structs, m)[4] == yoff[3]


def test_workspace_reused_across_shapes(tq, torch_cuda):
    """One workspace serves calls of different shapes in turn (the counter
    region is left zero by every call)."""
    import torch
    ws = tq.workspace(max(tq.tq_gemm_workspace(6144, 2560, 64), tq.tq_gemv_workspace(2560, 9728)))
    shapes = [(6144, 2560, 1), (2560, 9728, 1), (1024, 1536, 16), (6144, 2560, 64), (2560, 9728, 1)]
    for n, k, m in shapes:
        hw = host_weight(5, 0, 1, n, k)
        w = dev_weight(hw)
        if m == 1:
            x = torch.randn(k, device="cuda")
            y = tq.tq_gemv(w, x, ws=ws)
            ref = tq.tq_gemv(w, x)  # fresh zeroed workspace
        else:
            x = torch.randn((m, k), device="cuda").half()
            y = tq.tq_gemm(w, x, ws=ws)
            ref = tq.tq_gemm(w, x)
        torch.cuda.synchronize()
        assert torch.equal(y, ref), (n, k, m)
