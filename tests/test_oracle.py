"""Pins of the oracle against facts outside itself (CPU only).

Each test checks one oracle function against a published value, a library
routine, a closed form, an invariant or brute force, chosen so that a
plausible slip (dropped term, wrong sign or index, transposed operand, a
missing block reset, double rounding) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import scipy.linalg

import oracle
import tqsynth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ---- generator -------------------------------------------------------------------

def test_splitmix64_published_vector():
    want = [int(t[0], 16) for t in _golden_lines("splitmix64_state0.txt")]
    got = [oracle.draw(0, i) for i in range(4)]
    assert got == want


def test_stack_phase_seed_is_keyed_mix():
    # key(seed, tag) = mix64(seed ^ mix64(tag)); distinct per layer/phase
    seeds = {oracle.stack_phase_seed(0, l, p) for l in range(4) for p in range(4)}
    assert len(seeds) == 16
    tag = 0x516E0000 | (3 << 2) | 1
    assert oracle.stack_phase_seed(7, 3, 1) == oracle.mix64(7 ^ oracle.mix64(tag))


def test_rht_signs_balanced_and_from_top_bit():
    d = oracle.rht_signs(123, 4096)
    assert set(np.unique(d)) == {-1, 1}
    assert abs(d.mean()) < 0.06
    for k in (0, 1, 511, 4095):
        assert d[k] == (-1 if oracle.draw(123, k) >> 63 else 1)


# ---- rounding ----------------------------------------------------------------------

def _all_f16_in(lo, hi):
    b = np.arange(0, 0x7C00, dtype=np.uint16)
    v = b.view(np.float16).astype(np.float64)
    return b[(v >= lo) & (v <= hi)]


def test_f16_rounding_exhaustive_products_vs_numpy():
    """Every fp16 scale in [0.005, 0.03] times every component of the seed-0
    codebook: the oracle's fp16_RNE of the exact product equals numpy's."""
    sc = _all_f16_in(0.005, 0.03).view(np.float16).astype(np.float64)
    cb = tqsynth.codebook(0).reshape(-1).view(np.float16).astype(np.float64)
    prod = (sc[:, None] * cb[None, :]).ravel()  # exact: 11 x 11 bit significands
    want = prod.astype(np.float16).view(np.uint16)
    got = oracle.f16_from_f64(prod)
    assert np.array_equal(got, want)
    # the set covers fp16 subnormal results too
    assert np.any(np.abs(prod) < 2.0 ** -14)


def test_f16_rounding_ties_subnormals_overflow():
    ulp = 2.0 ** -10
    cases = [1.0 + ulp / 2, 1.0 + 1.5 * ulp, -(1.0 + ulp / 2), 2.0 ** -25, 3 * 2.0 ** -25,
             2.0 ** -24 * 1.5, 65504.0, 65519.99, 65520.0, 1e6, -1e6, 2.0 ** -14 - 2.0 ** -25,
             0.0, -0.0, 5.960464477539063e-08, 6.097555160522461e-05]
    rng = np.random.default_rng(1)
    rnd = rng.standard_normal(20000) * np.exp(rng.uniform(-20, 12, 20000))
    v = np.concatenate([np.array(cases), rnd])
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.f16_from_f64(v), want)


def _bf16_brute(x):
    """Nearest finite bf16 by scanning all of them; ties to the even code."""
    bits = np.arange(0, 0x7F80, dtype=np.uint32)
    vals = (bits << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    out = []
    for xv in x:
        ax = abs(xv)
        d = np.abs(vals - ax)
        m = d.min()
        idx = np.nonzero(d == m)[0]
        pick = idx[0] if len(idx) == 1 else [i for i in idx if (bits[i] & 1) == 0][0]
        out.append(int(bits[pick]) | (0x8000 if math.copysign(1, xv) < 0 else 0))
    return np.array(out, dtype=np.uint16)


def test_bf16_rounding_brute_force():
    rng = np.random.default_rng(2)
    x = rng.standard_normal(300) * np.exp(rng.uniform(-8, 8, 300))
    # exact ties: midpoints between adjacent bf16 values
    base = (np.array([0x3F80, 0x3F81, 0x4000, 0x4011, 0x3C00], dtype=np.uint32) << 16).view(np.float32)
    nxt = ((np.array([0x3F81, 0x3F82, 0x4001, 0x4012, 0x3C01], dtype=np.uint32)) << 16).view(np.float32)
    ties = (base.astype(np.float64) + nxt.astype(np.float64)) / 2
    x = np.concatenate([x, ties, -ties, [0.0, -0.0]])
    assert np.array_equal(oracle.bf16_from_f64(x), _bf16_brute(x))


def test_generator_bf16_matches_oracle_rounding():
    # the input module's bf16 conversion agrees with the oracle's on its draws
    z = tqsynth._normals(tqsynth.key(5, tqsynth.TAG_ACTIVATION), 0, 50000)
    assert np.array_equal(tqsynth.bf16_bits(z), oracle.bf16_from_f64(z))


# ---- decode ------------------------------------------------------------------------

def _hand_codebook():
    s = np.arange(8)[:, None, None]
    c = np.arange(256)[None, :, None]
    j = np.arange(4)[None, None, :]
    v = ((-1.0) ** j) * (2.0 ** (j >> 1)) * (s + c / 256.0)
    return v.astype(np.float16).view(np.uint16)


def test_decode_hand_example_single_block():
    rows = [t for t in _golden_lines("decode_hand_example.txt") if t[0] == "A"]
    codes = np.array([[int(t[2]) for t in rows]], dtype=np.uint8)
    scales = np.array([[np.float16(0.5).view(np.uint16)]], dtype=np.uint16)
    w = oracle.decode(codes, scales, _hand_codebook(), 1, 32)
    got = w.view(np.float16).astype(np.float64).reshape(8, 4)
    want = np.array([[float(v) for v in t[5:9]] for t in rows])
    assert np.array_equal(got, want)


def test_decode_hand_example_block_reset():
    rows = [t for t in _golden_lines("decode_hand_example.txt") if t[0] == "B"]
    codes = np.zeros((1, 128), dtype=np.uint8)
    for t in rows:
        codes[0, int(t[1])] = int(t[2])
    scales = np.array([[np.float16(1.0).view(np.uint16), np.float16(0.5).view(np.uint16)]], dtype=np.uint16)
    w = oracle.decode(codes, scales, _hand_codebook(), 1, 512).view(np.float16).astype(np.float64).reshape(128, 4)
    want = np.zeros((128, 4))
    for t in rows:
        want[int(t[1])] = [float(v) for v in t[5:9]]
    assert np.array_equal(w, want)


def test_decode_rows_matches_full_decode():
    n, k = 37, 1024
    c = tqsynth.codes(3, 0, 0, n, k)
    s = tqsynth.scales(3, 0, 0, n, k)
    cb = tqsynth.codebook(3)
    full = oracle.decode(c, s, cb, n, k)
    assert np.array_equal(oracle.decode_rows(c, s, cb, k, 5, 9), full[5:9])


def test_decode_state_uses_previous_code_low_bits():
    # a codebook that is zero except in state 5: only groups whose previous
    # code ends in binary 101 (and that are not at a block start) decode to
    # nonzero values
    cb = np.zeros((8, 256, 4), dtype=np.float16)
    cb[5] = 1.0
    codes = tqsynth.codes(9, 0, 0, 2, 512)
    scales = np.full((2, 2), np.float16(1.0).view(np.uint16), dtype=np.uint16)
    w = oracle.decode(codes, scales, cb.view(np.uint16), 2, 512).view(np.float16).reshape(2, 128, 4)
    prev = np.concatenate([np.zeros((2, 1), dtype=np.uint8), codes[:, :-1]], axis=1)
    expect = ((prev & 7) == 5)
    expect[:, 0] = False
    expect[:, 64] = False
    assert np.array_equal(w[:, :, 0] == 1.0, expect)


def test_size_arithmetic():
    # codes: 1 byte per 4 weights; scales: 2 bytes per 256 weights -> 33/128 B per weight
    for n, k in [(1024, 1024), (4096, 2560), (2560, 9728), (5120, 17408)]:
        c = tqsynth.codes(0, 0, 0, 8, k)  # row width only
        assert c.shape[1] * n == n * k // 4
        assert tqsynth.pack_bytes(n, k) * 128 == n * k * 33
    assert tqsynth.pack_bytes(1024, 1024) == 270336
    # 2 bits per weight alone is 87.5% smaller than 16 bits ("Size" section)
    assert 1 - 2 / 16 == 0.875
    assert abs(33 / 128 * 8 - 2.0625) < 1e-15


# ---- RHT ---------------------------------------------------------------------------------

def _rht_matrix(seed):
    eye = np.eye(512)
    return oracle.rht_f64(eye, 512, 512, seed).T  # column j = image of e_j


def test_rht_matrix_is_scipy_hadamard_times_signs():
    seed = 77
    T = _rht_matrix(seed)
    H = scipy.linalg.hadamard(512) / math.sqrt(512)
    d = oracle.rht_signs(seed, 512).astype(np.float64)
    assert np.max(np.abs(T - H * d[None, :])) < 1e-14
    assert np.max(np.abs(T @ T.T - np.eye(512))) < 1e-13
    Hn = T * d[None, :]  # strip D: H itself
    assert np.max(np.abs(Hn @ Hn - np.eye(512))) < 1e-13  # H is its own inverse


def test_rht_closed_forms_and_norm():
    seed, k = 11, 1024
    d = oracle.rht_signs(seed, k).astype(np.float64)
    # x = D 1  ->  D x = 1  ->  H 1 = sqrt(512) e_0 in every block
    y = oracle.rht_f64(d[None, :], 1, k, seed)[0]
    want = np.zeros(k)
    want[0] = want[512] = math.sqrt(512)
    assert np.max(np.abs(y - want)) < 1e-12
    # x = D e_0 -> H e_0 = 1/sqrt(512)
    e0 = np.zeros(k)
    e0[0] = d[0]
    y = oracle.rht_f64(e0[None, :], 1, k, seed)[0]
    assert np.max(np.abs(y[:512] - 1 / math.sqrt(512))) < 1e-15 and np.all(y[512:] == 0)
    # norms are kept block by block; the inverse is D H x'
    xb = tqsynth.activations(4, 3, k)
    x = tqsynth.bf16_to_f64(xb)
    xr = oracle.rht(xb, 3, k, seed)
    for b in range(2):
        assert np.allclose(np.linalg.norm(xr[:, 512 * b:512 * b + 512], axis=1),
                           np.linalg.norm(x[:, 512 * b:512 * b + 512], axis=1), rtol=1e-13)
    H = scipy.linalg.hadamard(512) / math.sqrt(512)
    back = np.concatenate([xr[:, :512] @ H, xr[:, 512:] @ H], axis=1) * d[None, :]
    assert np.max(np.abs(back - x)) < 1e-12


def test_rht_bf16_path_equals_f64_path():
    xb = tqsynth.activations(8, 2, 512)
    assert np.array_equal(oracle.rht(xb, 2, 512, 5), oracle.rht_f64(tqsynth.bf16_to_f64(xb), 2, 512, 5))


# ---- matmul ------------------------------------------------------------------------------

def test_matmul_vs_numpy_and_linearity():
    n, k, m = 24, 512, 3
    w = oracle.decode(tqsynth.codes(1, 0, 0, n, k), tqsynth.scales(1, 0, 0, n, k), tqsynth.codebook(1), n, k)
    rng = np.random.default_rng(0)
    x1, x2 = rng.standard_normal((m, k)), rng.standard_normal((m, k))
    y1 = oracle.matmul(w, x1, m, n, k)
    W = w.view(np.float16).astype(np.float64)
    assert np.allclose(y1, x1 @ W.T, rtol=1e-12, atol=1e-12)
    y12 = oracle.matmul(w, 2 * x1 - 3 * x2, m, n, k)
    assert np.allclose(y12, 2 * y1 - 3 * oracle.matmul(w, x2, m, n, k), rtol=1e-11, atol=1e-11)


def test_linear_constant_codebook_closed_form():
    # cb = 1 everywhere -> W[n][k] = scale[n][k/256] -> y = sum_b scale_b * sum(x' over block b)
    n, k = 5, 1024
    cb = np.full((8, 256, 4), np.float16(1.0)).view(np.uint16)
    codes = tqsynth.codes(2, 0, 0, n, k)
    sc = tqsynth.scales(2, 0, 0, n, k)
    xr = np.random.default_rng(3).standard_normal((1, k))
    y = oracle.linear(codes, sc, cb, n, k, xr, 1)[0]
    blocks = xr[0].reshape(4, 256).sum(axis=1)
    want = tqsynth.f16_to_f64(sc) @ blocks
    assert np.allclose(y, want, rtol=1e-13)


def test_linear_rows_matches_decode_then_numpy():
    n, k, m = 40, 1024, 2
    c, s, cb = tqsynth.codes(6, 1, 2, n, k), tqsynth.scales(6, 1, 2, n, k), tqsynth.codebook(6)
    xr = np.random.default_rng(4).standard_normal((m, k))
    W = oracle.decode(c, s, cb, n, k).view(np.float16).astype(np.float64)
    y = oracle.linear_rows(c, s, cb, k, xr, m, 7, 19)
    assert np.allclose(y, xr @ W[7:19].T, rtol=1e-12, atol=1e-12)


# ---- Viterbi ----------------------------------------------------------------------------

def _brute_min_cost(w, cb_bits, scale_bits, groups):
    sc = np.float64(np.uint16(scale_bits).view(np.float16))
    cbv = cb_bits.view(np.float16).astype(np.float64)
    dec = (sc * cbv).astype(np.float16).astype(np.float64)  # numpy's fp16 rounding: [8][256][4]
    W = w.reshape(groups, 4)
    E = [((W[g][None, None, :] - dec) ** 2).sum(axis=2) for g in range(groups)]  # [state][code]
    c = np.arange(256)
    if groups == 1:
        return E[0][0].min()
    if groups == 2:
        tot = E[0][0][:, None] + E[1][c & 7, :]
        return tot.min()
    tot = (E[0][0][:, None, None] + E[1][(c & 7)][:, :, None] + E[2][(c & 7)][None, :, :])
    return tot.min()


@pytest.mark.parametrize("groups", [1, 2, 3])
def test_viterbi_equals_brute_force(groups):
    cb = tqsynth.codebook(12)
    sc = np.array([np.float16(0.02).view(np.uint16)], dtype=np.uint16)
    rng = np.random.default_rng(groups)
    for _ in range(2):
        w = rng.standard_normal(4 * groups) * 0.02
        codes, cost = oracle.viterbi(w, 4 * groups, cb, sc)
        assert abs(cost - _brute_min_cost(w, cb, sc[0], groups)) <= 1e-15 * max(1.0, cost)
        assert abs(oracle.code_cost(w, 4 * groups, cb, sc, codes) - cost) <= 1e-18


def test_viterbi_round_trip_on_decodable_rows():
    k = 512
    cb = tqsynth.codebook(13)
    codes = tqsynth.codes(13, 0, 0, 1, k)
    sc = tqsynth.scales(13, 0, 0, 1, k)
    w = oracle.decode(codes, sc, cb, 1, k).view(np.float16).astype(np.float64)[0]
    enc, cost = oracle.viterbi(w, k, cb, sc[0])
    assert cost == 0.0
    assert np.array_equal(oracle.decode(enc[None, :], sc, cb, 1, k)[0].view(np.float16).astype(np.float64), w)


# ---- encoder with binary32 decisions -------------------------------------------------------

def _path_values(codes, cb_bits):
    """Unscaled codebook values along a code path of one 256-block (fp64 [256])."""
    cbv = cb_bits.view(np.float16).astype(np.float64).reshape(8, 256, 4)
    st = np.concatenate([[0], codes[:-1] & 7])
    return cbv[st, codes].reshape(-1)


@pytest.mark.parametrize("groups", [1, 2, 3])
def test_viterbi32_path_is_optimal_within_binary32(groups):
    # brute force over all 256^groups paths in binary64 (numpy fp16 rounding)
    cb = tqsynth.codebook(21)
    sc = np.float16(0.02).view(np.uint16)
    rng = np.random.default_rng(100 + groups)
    for _ in range(3):
        w = (rng.standard_normal(4 * groups) * 0.02).astype(np.float32)
        codes, j = oracle.viterbi32(w, groups, cb, sc)
        best = _brute_min_cost(w.astype(np.float64), cb, sc, groups)
        got = oracle.code_cost(w.astype(np.float64), 4 * groups, cb, np.array([sc], np.uint16), codes)
        wn = float((w.astype(np.float64) ** 2).sum())
        assert got - best <= 1e-5 * wn
        # the returned cost is the squared error minus |w|^2
        assert abs((j + wn) - got) <= 1e-5 * wn


def test_viterbi32_agrees_with_binary64_viterbi_on_blocks():
    cb = tqsynth.codebook(22)
    rng = np.random.default_rng(5)
    same = 0
    for trial in range(6):
        w = rng.standard_normal(256).astype(np.float32)
        sc = np.float16([0.8, 1.0, 1.2][trial % 3]).view(np.uint16)
        c32, j32 = oracle.viterbi32(w, 64, cb, sc)
        c64, cost64 = oracle.viterbi(w.astype(np.float64), 256, cb, np.array([sc], np.uint16))
        cost32 = oracle.code_cost(w.astype(np.float64), 256, cb, np.array([sc], np.uint16), c32)
        assert cost32 - cost64 <= 1e-5 * float((w.astype(np.float64) ** 2).sum())
        same += int(np.array_equal(c32, c64))
    assert same >= 4  # identical paths except on near-ties


def test_viterbi32_round_trip_on_decodable_block():
    cb = tqsynth.codebook(23)
    codes = tqsynth.codes(23, 0, 0, 1, 256)[0]
    sc = np.float16(0.75).view(np.uint16)
    w = oracle.decode(codes[None, :], np.array([[sc]], np.uint16), cb, 1, 256).view(np.float16)
    w = w.astype(np.float32)[0]
    enc, j = oracle.viterbi32(w, 64, cb, sc)
    cost = oracle.code_cost(w.astype(np.float64), 256, cb, np.array([sc], np.uint16), enc)
    assert cost == 0.0
    assert abs(j + float((w.astype(np.float64) ** 2).sum())) <= 1e-4


@pytest.mark.parametrize("lam,bits", [(0.5, 0x3800), (0.125, 0x3000), (-0.25, 0xB400), (2.0, 0x4000)])
def test_refit32_exact_for_power_of_two_multiples(lam, bits):
    # w = lam * e with lam a power of two: sum w*e = lam * sum e*e exactly
    cb = tqsynth.codebook(24)
    codes = tqsynth.codes(24, 0, 0, 1, 256)[0]
    w = (lam * _path_values(codes, cb)).astype(np.float32)
    assert oracle.refit32(w, codes, cb) == bits


def test_refit32_none_without_energy():
    cb = np.zeros(8 * 256 * 4, dtype=np.uint16)  # all-zero codebook
    w = np.ones(256, dtype=np.float32)
    assert oracle.refit32(w, np.zeros(64, np.uint8), cb) is None


@pytest.mark.parametrize("gain,bits", [(0.5, 0x3E00), (0.25, 0x3A00)])
def test_encode32_initial_scale_closed_form(gain, bits):
    # |w| = 3 everywhere: RMS = 3 exactly, scale = fp16(3 * gain)
    rng = np.random.default_rng(3)
    w = (3.0 * rng.choice([-1.0, 1.0], size=(2, 512))).astype(np.float32)
    _, scales, _ = oracle.encode32(w, tqsynth.codebook(25), gain, 0)
    assert (scales == bits).all()


def test_encode32_zero_block():
    w = np.zeros((1, 512), dtype=np.float32)
    codes, scales, err = oracle.encode32(w, tqsynth.codebook(26), 1.0, 2)
    assert (codes == 0).all() and (scales == 0).all() and (err == 0).all()


def test_encode32_err_is_decoded_squared_error():
    cb = tqsynth.codebook(27)
    w = np.random.default_rng(8).standard_normal((3, 768)).astype(np.float32)
    codes, scales, err = oracle.encode32(w, cb, 1.0, 1)
    wh = oracle.decode(codes, scales, cb, 3, 768).view(np.float16).astype(np.float64)
    want = ((w.astype(np.float64) - wh) ** 2).reshape(3, 3, 256).sum(axis=2)
    assert np.allclose(err, want, rtol=1e-5, atol=0)


def test_encode32_refits_never_increase_error():
    cb = tqsynth.codebook(28)
    w = np.random.default_rng(9).standard_normal((2, 1024)).astype(np.float32)
    prev = None
    for r in range(4):
        _, _, err = oracle.encode32(w, cb, 1.0, r)
        if prev is not None:
            assert (err <= prev * (1 + 1e-6)).all()
        prev = err


def test_encode32_gaussian_mse_between_bounds():
    # Unit Gaussian weights at 2.0625 bits per weight: the distortion-rate
    # bound is 2^(-2R); the best 2-bit scalar quantizer (Lloyd-Max, 4 levels)
    # reaches 0.1175 (Max 1960).  The trellis must land between the two.
    cb = tqsynth.codebook(0)
    gain = 1.0 / math.sqrt(float((cb.view(np.float16).astype(np.float64) ** 2).mean()))
    w = np.random.default_rng(11).standard_normal((4, 1024)).astype(np.float32)
    _, _, err = oracle.encode32(w, cb, gain, 1)
    mse = float(err.astype(np.float64).sum()) / w.size
    assert 2.0 ** (-2 * 2.0625) < mse < 0.1175


# ---- block LDLQ ------------------------------------------------------------------------------

def _cb_gain(seed):
    cb = tqsynth.codebook(seed)
    return cb, float(np.float32(1.0 / math.sqrt(float((cb.view(np.float16).astype(np.float64) ** 2).mean()))))


def _proxy_loss(w, codes, scales, cb, u):
    n, k = w.shape
    wh = oracle.decode(codes, scales, cb, n, k).view(np.float16).astype(np.float64)
    e = w.astype(np.float64) - wh
    return float(((e @ (np.eye(k) + u.astype(np.float64))) ** 2).sum())


def test_ldlq_without_feedback_is_the_plain_encoder():
    cb, g = _cb_gain(30)
    w = tqsynth.weight_rows_f32(30, 5, 1024)
    got = oracle.ldlq32(w, np.zeros((1024, 1024), np.float32), cb, g, 1)
    want = oracle.encode32(w, cb, g, 1)
    for a, b in zip(got, want):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("gamma", [0.5, 2.0])
def test_ldlq_proxy_loss_identity(gamma):
    # H = (I+U)(I+U)^T: tr(E H E^T) = |E (I+U)|^2 must equal the summed squared
    # errors of the adjusted blocks (the feedback cancels the earlier errors
    # exactly); a wrong sign, a transposed U or feeding the adjusted-block error
    # instead of E breaks it
    cb, g = _cb_gain(31)
    w = tqsynth.weight_rows_f32(31, 6, 1536)
    u = tqsynth.hessian_factor(31, 1536, gamma)
    codes, scales, err = oracle.ldlq32(w, u, cb, g, 1)
    loss = _proxy_loss(w, codes, scales, cb, u)
    assert abs(loss - float(err.astype(np.float64).sum())) <= 1e-5 * loss


def test_ldlq_lowers_the_proxy_loss():
    cb, g = _cb_gain(32)
    w = tqsynth.weight_rows_f32(32, 8, 1024)
    u = tqsynth.hessian_factor(32, 1024, 0.5)
    c1, s1, _ = oracle.ldlq32(w, u, cb, g, 1)
    c0, s0, _ = oracle.encode32(w, cb, g, 1)
    assert _proxy_loss(w, c1, s1, cb, u) < 0.95 * _proxy_loss(w, c0, s0, cb, u)


def test_hessian_factor_is_block_strictly_upper():
    u = tqsynth.hessian_factor(33, 1024)
    bi = np.arange(1024) // 256
    assert (u[bi[:, None] >= bi[None, :]] == 0).all()
    assert (u[bi[:, None] < bi[None, :]] != 0).all()


# ---- stack -------------------------------------------------------------------------------

@pytest.mark.parametrize("p", [0, 1, 2, 3])
def test_stack_phase_constant_codebook_closed_form(p):
    # Every codebook entry 1 and one scale per row: W[n][k] = s_n, and the
    # Sylvester Hadamard's columns sum to 0 except the first, so each 512-block
    # of x' sums to sqrt(512) d_0 x_0 and y_n = s_n sqrt(512) sum_B d_512B x_512B.
    # Pins the phase composition: the RHT seed, every op of the phase, and
    # which op feeds the bf16 handoff with which alpha.
    m, k = 2, 1024
    seed = 4242
    cb = np.full(8 * 256 * 4, np.float16(1.0).view(np.uint16), dtype=np.uint16)
    rng = np.random.default_rng(p)
    ops = oracle.PHASES[p]
    weights = {}
    for i, op in enumerate(ops):
        n = 48 + 16 * i
        s_row = (0.005 + 0.025 * rng.random(n)).astype(np.float16)
        scales = np.repeat(s_row.view(np.uint16)[:, None], k // 256, axis=1)
        codes = rng.integers(0, 256, size=(n, k // 4), dtype=np.uint8)
        weights[op] = (codes, scales, cb, n, k)
    x = tqsynth.activations(p + 7, m, k)
    ys, hand = oracle.stack_phase(p, x, m, weights, seed)
    d = oracle.rht_signs(seed, k).astype(np.float64)
    xv = tqsynth.bf16_to_f64(x)
    col = (xv[:, ::512] * d[::512]).sum(axis=1) * math.sqrt(512.0)  # [m]
    for op in ops:
        s_row = tqsynth.f16_to_f64(weights[op][1][:, 0])
        want = col[:, None] * s_row[None, :]
        assert np.allclose(ys[op], want, rtol=1e-12, atol=1e-15)
    hop = oracle.HANDOFF_OP[p]
    assert hop == ops[0]
    want_h = tqsynth.bf16_bits(oracle.alpha(k) * ys[hop])
    assert np.array_equal(hand, want_h)


def _signs_from_definition(seed_lp: int, k: int) -> np.ndarray:
    """d[j] = -1 when the top bit of the j-th SplitMix64 output (state seed_lp)
    is set, from the input generator's SplitMix64 (not the oracle's)."""
    return np.where(tqsynth.draws(seed_lp, 0, k) >> np.uint64(63), -1.0, 1.0)


def _phase_seed_from_definition(seed: int, l: int, p: int) -> int:
    return tqsynth.mix64_int(seed ^ tqsynth.mix64_int(0x516E0000 | (l << 2) | p))


def test_layer_stack_constant_codebook_closed_form_chain():
    # Three layers with every codebook entry 1 and one fp16 scale per row.
    # Then W = s_n, each phase's outputs are y_n = s_n * c with
    # c = sqrt(512) * sum_B d[512B] x[512B] (x = the phase input, d = that
    # phase's signs), and the whole stack collapses to a scalar recurrence on
    # the handoff op's row scales.  A wrong per-(layer, phase) seed, a phase
    # reading the wrong input, the wrong op handed on, or alpha of the wrong
    # width changes the chain.
    m, seed = 2, 987654321
    hidden, q, kv, inter = 1024, 512, 512, 1536
    shape = tqsynth.StackShape("chain", 3, hidden, q, kv, inter)
    cb = np.full((8, 256, 4), np.float16(1.0).view(np.uint16), dtype=np.uint16)
    rng = np.random.default_rng(77)
    layers = []
    for _ in range(shape.layers):
        w = {}
        for op, n, k in shape.ops():
            s_row = (0.005 + 0.025 * rng.random(n)).astype(np.float16).view(np.uint16)
            scales = np.repeat(s_row[:, None], k // 256, axis=1)
            codes = rng.integers(0, 256, size=(n, k // 4), dtype=np.uint8)
            w[op] = (codes, scales, cb, n, k)
        layers.append(w)
    x = tqsynth.activations(55, m, hidden)
    h_out, trace = oracle.layer_stack(layers, x, m, seed)
    assert len(trace) == 4 * shape.layers

    handoff_op = {0: "q", 1: "o", 2: "gate", 3: "down"}
    h = tqsynth.bf16_to_f64(x)  # [m][k] values of the current phase input
    f = 0
    for l, w in enumerate(layers):
        for p in range(4):
            op = handoff_op[p]
            n, k = w[op][3], w[op][4]
            assert k == h.shape[1]
            d = _signs_from_definition(_phase_seed_from_definition(seed, l, p), k)
            c = math.sqrt(512.0) * (h[:, ::512] * d[::512]).sum(axis=1)  # [m]
            s_row = tqsynth.f16_to_f64(w[op][1][:, 0])
            a = 1.0 / math.sqrt(k * (0.03 ** 3 - 0.005 ** 3) / (3 * 0.025))
            want = tqsynth.bf16_bits(a * (c[:, None] * s_row[None, :]))
            assert np.array_equal(trace[f], want), (l, p)
            h = tqsynth.bf16_to_f64(want)
            f += 1
    assert np.array_equal(h_out, trace[-1])


def test_stack_phase_seeds_differ_per_layer_and_phase():
    seeds = {oracle.stack_phase_seed(3, l, p) for l in range(8) for p in range(4)}
    assert len(seeds) == 32
    assert oracle.stack_phase_seed(3, 2, 1) == _phase_seed_from_definition(3, 2, 1)


def test_alpha_second_moment_closed_form():
    a, b = oracle.SCALE_LO, oracle.SCALE_HI
    assert abs(oracle.E_S2 - (a * a + a * b + b * b) / 3) < 1e-18
    assert abs(oracle.alpha(2560) - 1 / math.sqrt(2560 * 3.5833333333333e-4)) < 1e-9


def test_handoff_is_near_unit_variance():
    n, k = 256, 2560
    c, s, cb = tqsynth.codes(0, 0, 0, n, k), tqsynth.scales(0, 0, 0, n, k), tqsynth.codebook(0)
    x = tqsynth.activations(0, 1, k)
    xr = oracle.rht(x, 1, k, 1)
    y = oracle.linear(c, s, cb, n, k, xr, 1)
    h = tqsynth.bf16_to_f64(oracle.handoff(y, k))
    assert 0.8 < h.std() < 1.2


def test_rel_err_metric():
    r = np.array([1.0, -2.0, 0.0, 4.0])
    assert oracle.rel_err(r, r) == 0.0
    y = r + np.array([0.0, 0.0, 0.01, 0.0])
    rms = math.sqrt((1 + 4 + 0 + 16) / 4)
    assert abs(oracle.rel_err(y, r) - 0.01 / rms) < 1e-15
