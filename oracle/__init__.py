"""The oracle: plain fp64 CPU restatement of the trellis-decode matmul path.

TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the benchmark's
CPU-baseline leg may import this package.  It never imports the CUDA
library and the CUDA library never imports it; both take their inputs from
``tqsynth``.

The arithmetic lives in ``tq_oracle.c`` (plain C, binary64, compiled with
``-O2 -ffp-contract=off``, no fast-math); this file loads it with ctypes and
adds the layer-stack composition, which only chains the C functions.

Pages (cited by title and section):
  * "Pingala-8" landing page, "How it works": 8-state trellis code over
    groups of 4 weights; random Hadamard rotation before encoding.
  * "Bonsai 2 27B" article, change of basis: the rotation is folded into the
    weights and the matching transform is applied to the activations.
  * "8 open models ... what 2-bit quantization costs", "Size": per-block
    scales add bits on top of the 2-bit codes.

Readings where the pages are silent:
  * layout: codes uint8 [n][k/4]; state = previous code & 7, reset every
    256 weights; fp16 scale per (row, 256-block); codebook fp16 [8][256][4];
    component j of an entry is weight 4g+j.
  * decode rounds once: fp16_RNE(scale * cb), subnormals kept.
  * RHT: D first, then H_512 in natural (Sylvester) order, /sqrt(512).
  * layer stack: handoff = bf16_RNE(alpha(k) * y) with
    alpha(k) = 1/sqrt(k * E[s^2]), E[s^2] = (0.03^3 - 0.005^3)/(3*0.025).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq_oracle.c")
_LIB = os.path.join(_HERE, "libtq_oracle.so")
CFLAGS = ["-O2", "-ffp-contract=off", "-fPIC", "-shared", "-Wall"]


def build(force: bool = False) -> str:
    """Compile tq_oracle.c into libtq_oracle.so next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", *CFLAGS, "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        u8p, u16p, f64p = (ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(ctypes.c_uint16),
                           ctypes.POINTER(ctypes.c_double))
        i64, u64 = ctypes.c_int64, ctypes.c_uint64
        L.orc_mix64.restype = u64
        L.orc_mix64.argtypes = [u64]
        L.orc_draw.restype = u64
        L.orc_draw.argtypes = [u64, u64]
        L.orc_rht_sign.restype = ctypes.c_int
        L.orc_rht_sign.argtypes = [u64, i64]
        L.orc_stack_phase_seed.restype = u64
        L.orc_stack_phase_seed.argtypes = [u64, ctypes.c_int32, ctypes.c_int32]
        L.orc_f16_to_f64.restype = ctypes.c_double
        L.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_f64.restype = ctypes.c_double
        L.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_f16_from_f64.restype = ctypes.c_uint16
        L.orc_f16_from_f64.argtypes = [ctypes.c_double]
        L.orc_bf16_from_f64.restype = ctypes.c_uint16
        L.orc_bf16_from_f64.argtypes = [ctypes.c_double]
        L.orc_f16_from_f64_array.argtypes = [f64p, i64, u16p]
        L.orc_bf16_from_f64_array.argtypes = [f64p, i64, u16p]
        L.orc_decode.argtypes = [u8p, u16p, u16p, i64, i64, u16p]
        L.orc_decode_rows.argtypes = [u8p, u16p, u16p, i64, i64, i64, u16p]
        L.orc_rht.argtypes = [u16p, i64, i64, u64, f64p]
        L.orc_rht_f64.argtypes = [f64p, i64, i64, u64, f64p]
        L.orc_matmul.argtypes = [u16p, f64p, i64, i64, i64, f64p]
        L.orc_linear_rows.argtypes = [u8p, u16p, u16p, i64, f64p, i64, i64, i64, f64p]
        L.orc_viterbi.restype = ctypes.c_double
        L.orc_viterbi.argtypes = [f64p, i64, u16p, u16p, u8p]
        L.orc_code_cost.restype = ctypes.c_double
        L.orc_code_cost.argtypes = [f64p, i64, u16p, u16p, u8p]
        f32p = ctypes.POINTER(ctypes.c_float)
        L.orc_viterbi32.restype = ctypes.c_float
        L.orc_viterbi32.argtypes = [f32p, ctypes.c_int, u16p, ctypes.c_uint16, u8p]
        L.orc_refit32.restype = ctypes.c_int
        L.orc_refit32.argtypes = [f32p, u8p, u16p, u16p]
        L.orc_encode32.argtypes = [f32p, i64, i64, u16p, ctypes.c_float, ctypes.c_int, u8p, u16p, f32p]
        L.orc_ldlq32.argtypes = [f32p, i64, i64, f32p, u16p, ctypes.c_float, ctypes.c_int, u8p, u16p, f32p]
        _lib = L
    return _lib


def _p(a: np.ndarray, ct):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _c(a, dtype):
    return np.ascontiguousarray(np.asarray(a, dtype=dtype))


# ---- generator (SplitMix64) -------------------------------------------------

def mix64(z: int) -> int:
    return int(lib().orc_mix64(z))


def draw(key: int, i: int) -> int:
    return int(lib().orc_draw(key, i))


def rht_signs(seed: int, k: int) -> np.ndarray:
    L = lib()
    return np.array([L.orc_rht_sign(seed, i) for i in range(k)], dtype=np.int8)


def stack_phase_seed(seed: int, layer: int, phase: int) -> int:
    return int(lib().orc_stack_phase_seed(seed, layer, phase))


# ---- rounding -----------------------------------------------------------------

def f16_from_f64(v) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().orc_f16_from_f64_array(_p(v, ctypes.c_double), v.size, _p(out, ctypes.c_uint16))
    return out


def bf16_from_f64(v) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().orc_bf16_from_f64_array(_p(v, ctypes.c_double), v.size, _p(out, ctypes.c_uint16))
    return out


def f16_to_f64(bits) -> np.ndarray:
    L = lib()
    b = _c(bits, np.uint16)
    return np.array([L.orc_f16_to_f64(int(x)) for x in b.ravel()], dtype=np.float64).reshape(b.shape)


def bf16_to_f64(bits) -> np.ndarray:
    L = lib()
    b = _c(bits, np.uint16)
    return np.array([L.orc_bf16_to_f64(int(x)) for x in b.ravel()], dtype=np.float64).reshape(b.shape)


# ---- the path -------------------------------------------------------------------

def decode(codes, scales, codebook, n: int, k: int) -> np.ndarray:
    """fp16 bits [n][k] of the decoded weight."""
    codes, scales, codebook = _c(codes, np.uint8), _c(scales, np.uint16), _c(codebook, np.uint16)
    out = np.empty((n, k), dtype=np.uint16)
    lib().orc_decode(_p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint16), _p(codebook, ctypes.c_uint16),
                     n, k, _p(out, ctypes.c_uint16))
    return out


def decode_rows(codes, scales, codebook, k: int, row_begin: int, row_end: int) -> np.ndarray:
    codes, scales, codebook = _c(codes, np.uint8), _c(scales, np.uint16), _c(codebook, np.uint16)
    out = np.empty((row_end - row_begin, k), dtype=np.uint16)
    lib().orc_decode_rows(_p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint16), _p(codebook, ctypes.c_uint16),
                          k, row_begin, row_end, _p(out, ctypes.c_uint16))
    return out


def rht(x_bf16, m: int, k: int, seed: int) -> np.ndarray:
    """fp64 [m][k] = H_512 D x blockwise, from bf16 bits."""
    x = _c(x_bf16, np.uint16)
    out = np.empty((m, k), dtype=np.float64)
    lib().orc_rht(_p(x, ctypes.c_uint16), m, k, seed, _p(out, ctypes.c_double))
    return out


def rht_f64(x, m: int, k: int, seed: int) -> np.ndarray:
    x = _c(x, np.float64)
    out = np.empty((m, k), dtype=np.float64)
    lib().orc_rht_f64(_p(x, ctypes.c_double), m, k, seed, _p(out, ctypes.c_double))
    return out


def matmul(w_f16, xr, m: int, n: int, k: int) -> np.ndarray:
    """fp64 [m][n] = x' W^T with W fp16 bits [n][k] and x' fp64 [m][k]."""
    w, xr = _c(w_f16, np.uint16), _c(xr, np.float64)
    out = np.empty((m, n), dtype=np.float64)
    lib().orc_matmul(_p(w, ctypes.c_uint16), _p(xr, ctypes.c_double), m, n, k, _p(out, ctypes.c_double))
    return out


def linear_rows(codes, scales, codebook, k: int, xr, m: int, row_begin: int, row_end: int) -> np.ndarray:
    """fp64 [m][row_end-row_begin]: decode + matmul of the given rows only.
    `codes`/`scales` hold the full matrix (or at least rows < row_end)."""
    codes, scales, codebook = _c(codes, np.uint8), _c(scales, np.uint16), _c(codebook, np.uint16)
    xr = _c(xr, np.float64)
    out = np.empty((m, row_end - row_begin), dtype=np.float64)
    lib().orc_linear_rows(_p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint16), _p(codebook, ctypes.c_uint16),
                          k, _p(xr, ctypes.c_double), m, row_begin, row_end, _p(out, ctypes.c_double))
    return out


def linear(codes, scales, codebook, n: int, k: int, xr, m: int) -> np.ndarray:
    return linear_rows(codes, scales, codebook, k, xr, m, 0, n)


def viterbi(w, k: int, codebook, scales):
    """(codes uint8 [k/4], minimum cost) for one row."""
    w, codebook, scales = _c(w, np.float64), _c(codebook, np.uint16), _c(scales, np.uint16)
    codes = np.zeros(k // 4, dtype=np.uint8)
    cost = lib().orc_viterbi(_p(w, ctypes.c_double), k, _p(codebook, ctypes.c_uint16),
                             _p(scales, ctypes.c_uint16), _p(codes, ctypes.c_uint8))
    return codes, float(cost)


def code_cost(w, k: int, codebook, scales, codes) -> float:
    w, codebook, scales, codes = (_c(w, np.float64), _c(codebook, np.uint16), _c(scales, np.uint16),
                                  _c(codes, np.uint8))
    return float(lib().orc_code_cost(_p(w, ctypes.c_double), k, _p(codebook, ctypes.c_uint16),
                                     _p(scales, ctypes.c_uint16), _p(codes, ctypes.c_uint8)))


# ---- encoder with binary32 decisions -------------------------------------------

def viterbi32(w, groups: int, codebook, scale_bits: int):
    """(codes uint8 [groups], least path cost) of the binary32 Viterbi over
    `groups` groups of w (fp32) at one fp16 scale."""
    w, codebook = _c(w, np.float32), _c(codebook, np.uint16)
    codes = np.zeros(groups, dtype=np.uint8)
    j = lib().orc_viterbi32(_p(w, ctypes.c_float), groups, _p(codebook, ctypes.c_uint16), int(scale_bits),
                            _p(codes, ctypes.c_uint8))
    return codes, float(j)


def refit32(w, codes, codebook):
    """Least-squares fp16 scale bits of one 256-weight block for fixed codes,
    or None when there is none."""
    w, codes, codebook = _c(w, np.float32), _c(codes, np.uint8), _c(codebook, np.uint16)
    out = np.zeros(1, dtype=np.uint16)
    ok = lib().orc_refit32(_p(w, ctypes.c_float), _p(codes, ctypes.c_uint8), _p(codebook, ctypes.c_uint16),
                           _p(out, ctypes.c_uint16))
    return int(out[0]) if ok else None


def encode32(w, codebook, gain: float, refits: int):
    """Encode rotated weights w fp32 [n][k] (k % 256 == 0): (codes uint8
    [n][k/4], scales fp16 bits [n][k/256], err fp32 [n][k/256])."""
    w = _c(w, np.float32)
    n, k = w.shape
    codebook = _c(codebook, np.uint16)
    codes = np.zeros((n, k // 4), dtype=np.uint8)
    scales = np.zeros((n, k // 256), dtype=np.uint16)
    err = np.zeros((n, k // 256), dtype=np.float32)
    lib().orc_encode32(_p(w, ctypes.c_float), n, k, _p(codebook, ctypes.c_uint16), float(gain), int(refits),
                       _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint16), _p(err, ctypes.c_float))
    return codes, scales, err


def ldlq32(w, u, codebook, gain: float, refits: int):
    """Block LDLQ encoding of rotated weights w fp32 [n][k] with the Hessian
    factor u fp32 [k][k] (block strictly upper): (codes, scales, err) as
    encode32, err = per-block squared error of the adjusted blocks."""
    w, u = _c(w, np.float32), _c(u, np.float32)
    n, k = w.shape
    codebook = _c(codebook, np.uint16)
    codes = np.zeros((n, k // 4), dtype=np.uint8)
    scales = np.zeros((n, k // 256), dtype=np.uint16)
    err = np.zeros((n, k // 256), dtype=np.float32)
    lib().orc_ldlq32(_p(w, ctypes.c_float), n, k, _p(u, ctypes.c_float), _p(codebook, ctypes.c_uint16), float(gain),
                     int(refits), _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint16), _p(err, ctypes.c_float))
    return codes, scales, err


# ---- layer stack (composition of the functions above) ------------------------

SCALE_LO, SCALE_HI = 0.005, 0.03
E_S2 = (SCALE_HI ** 3 - SCALE_LO ** 3) / (3.0 * (SCALE_HI - SCALE_LO))  # E[s^2], s ~ U[lo, hi]


def alpha(k: int) -> float:
    """Handoff gain after an op with k inputs: 1/sqrt(k E[s^2]) keeps the
    next activation near unit variance (E[cb^2] = E[x'^2] = 1)."""
    return 1.0 / math.sqrt(k * E_S2)


def handoff(y: np.ndarray, k: int) -> np.ndarray:
    """bf16 bits of alpha(k) * y."""
    return bf16_from_f64(alpha(k) * np.asarray(y, dtype=np.float64))


# phase p of a layer: (ops computed, op whose output is handed on, its k)
PHASES = (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))
HANDOFF_OP = ("q", "o", "gate", "down")


def stack_phase(p: int, x_bf16: np.ndarray, m: int, weights: dict, seed_lp: int):
    """One phase: RHT of the bf16 input, then every op of the phase.
    weights[op] = (codes, scales, codebook, n, k).  Returns (ys, handoff bits)."""
    k = weights[PHASES[p][0]][4]
    xr = rht(x_bf16, m, k, seed_lp)
    ys = {}
    for op in PHASES[p]:
        c, s, cb, n, kk = weights[op]
        ys[op] = linear(c, s, cb, n, kk, xr, m)
    hop = HANDOFF_OP[p]
    return ys, handoff(ys[hop], weights[hop][4])


def layer_stack(layers: list, h_bf16: np.ndarray, m: int, seed: int):
    """Full stack: layers[l] = weights dict for layer l.  Returns the final
    bf16 hidden state and the list of per-phase handoffs."""
    h = _c(h_bf16, np.uint16)
    trace = []
    for l, w in enumerate(layers):
        for p in range(4):
            _, h = stack_phase(p, h, m, w, stack_phase_seed(seed, l, p))
            trace.append(h)
    return h, trace


def rel_err(y, yref) -> float:
    """max_i |y_i - ref_i| / max(|ref_i|, rms(ref)) over the tensor."""
    y = np.asarray(y, dtype=np.float64).ravel()
    r = np.asarray(yref, dtype=np.float64).ravel()
    if r.size == 0:
        return 0.0
    rms = math.sqrt(float(np.mean(r * r)))
    den = np.maximum(np.abs(r), rms)
    den = np.where(den == 0, 1.0, den)
    return float(np.max(np.abs(y - r) / den))
