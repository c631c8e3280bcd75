"""Seeded synthetic inputs for the trellis-decode matmul (shared by both sides).

This module is the only code that the CUDA path's tests/benchmark and the
oracle have in common.  It produces *inputs* -- trellis code bytes, fp16
block scales, the fp16 codebook set and bf16 activations -- and holds none
of the method's arithmetic (no decode, no transform, no matmul).

Generator: SplitMix64 (Steele, Lea & Flood 2014; Vigna's public reference),
used as a counter-based stream: draw(key, i) = mix64(key + (i+1)*gamma), the
i-th output of a SplitMix64 generator whose state starts at `key`.  Streams
are keyed per tensor: key(seed, tag) = mix64(seed ^ mix64(tag)).

Distributions (the pages train on real models; these seeded stand-ins have
the shapes of the pages' workloads -- Qwen3-4B, Llama-3.1-8B and a 27B-class
stack -- and the value ranges of the format):
  codes      uniform bytes; code t is byte (t mod 8) (little-endian) of draw(key, t // 8)
  scales     fp16_RNE(0.005 + 0.025*u), u = (draw >> 11) * 2^-53 (U[0.005, 0.03])
  codebook   fp16_RNE(z), z ~ N(0,1) by Box-Muller, [8][256][4]
  x          bf16_RNE(z), z ~ N(0,1) by Box-Muller, [m][k]
  dense W    bf16_RNE(std * z * (gain if u < rate else 1)), [n][k]: unquantized
             weight rows for the encoder (z ~ N(0,1); u a second uniform stream
             marks outliers)
  W rows     fp32_RNE(std * z), [n][k]: stand-in for already rotated weights
  Hessian    the factor U of H = (I + U)(I + U)^T, fp32 [k][k]: U[i][j] =
             gamma * z / sqrt(256 * (j // 256)) when i // 256 < j // 256, else 0
             (block strictly upper, each column's feedback of norm ~gamma)
Box-Muller for element t: u1 = ((draw(2t) >> 11) + 1) * 2^-53,
u2 = (draw(2t+1) >> 11) * 2^-53, z = sqrt(-2 ln u1) * cos(2 pi u2).
"""
from __future__ import annotations

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15

# op index inside one transformer layer: q, k, v, o, gate, up, down
OPS = ("q", "k", "v", "o", "gate", "up", "down")

TAG_CODEBOOK = 0xC0DEB00C
TAG_ACTIVATION = 0xAC7
TAG_DENSE = 0xDE45E000


def mix64_int(z: int) -> int:
    """SplitMix64 output mix on one Python int (mod 2^64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def key(seed: int, tag: int) -> int:
    return mix64_int((seed & MASK64) ^ mix64_int(tag))


def draws(k: int, start: int, count: int) -> np.ndarray:
    """draw(k, i) for i in [start, start+count), as uint64."""
    idx = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(np.uint64(k & MASK64) + (idx + np.uint64(1)) * np.uint64(GAMMA))


def _unit(r: np.ndarray) -> np.ndarray:
    return (r >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def _normals(k: int, start: int, count: int) -> np.ndarray:
    r = draws(k, 2 * start, 2 * count)
    r1, r2 = r[0::2], r[1::2]
    u1 = ((r1 >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
    u2 = _unit(r2)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def f16_bits(v: np.ndarray) -> np.ndarray:
    """fp64 -> IEEE binary16 bits (numpy's conversion rounds to nearest even)."""
    return np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)


def bf16_bits(v: np.ndarray) -> np.ndarray:
    """fp64 -> bfloat16 bits, round to nearest even, for finite values in the
    bf16 normal range (all that the generator produces) and zero."""
    v = np.asarray(v, dtype=np.float64)
    b = v.view(np.uint64)
    sign = ((b >> np.uint64(48)) & np.uint64(0x8000)).astype(np.uint32)
    mag = b & np.uint64(0x7FFFFFFFFFFFFFFF)
    top = (mag >> np.uint64(45)).astype(np.int64)  # 11 exponent + 7 mantissa bits
    low = (mag & np.uint64((1 << 45) - 1)).astype(np.int64)
    half = 1 << 44
    up = (low > half) | ((low == half) & ((top & 1) == 1))
    top = top + up.astype(np.int64)
    exp_d = top >> 7
    exp_b = exp_d - 1023 + 127
    zero = mag == 0
    if np.any(~zero & ((exp_b < 1) | (exp_b > 254))):
        raise ValueError("bf16_bits: value outside the bf16 normal range")
    out = (exp_b << 7) | (top & 0x7F)
    out = np.where(zero, 0, out).astype(np.uint32) | sign
    return out.astype(np.uint16)


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def weight_tag(layer: int, op: int, kind: int) -> int:
    return (layer << 8) | (op << 4) | kind


def codes(seed: int, layer: int, op: int, n: int, k: int) -> np.ndarray:
    """uint8 [n][k/4] uniform code bytes."""
    total = n * (k // 4)
    kk = key(seed, weight_tag(layer, op, 0))
    r = draws(kk, 0, (total + 7) // 8)
    return r.view(np.uint8)[:total].reshape(n, k // 4).copy()


def codes_rows(seed: int, layer: int, op: int, k: int, row_begin: int, row_end: int) -> np.ndarray:
    """The rows [row_begin, row_end) of codes(...), without generating the rest."""
    g = k // 4
    t0, t1 = row_begin * g, row_end * g
    kk = key(seed, weight_tag(layer, op, 0))
    d0 = t0 // 8
    r = draws(kk, d0, (t1 + 7) // 8 - d0)
    return r.view(np.uint8)[t0 - 8 * d0:t1 - 8 * d0].reshape(row_end - row_begin, g).copy()


def scales(seed: int, layer: int, op: int, n: int, k: int) -> np.ndarray:
    """fp16 bits [n][k/256], U[0.005, 0.03]."""
    nb = n * (k // 256)
    u = _unit(draws(key(seed, weight_tag(layer, op, 1)), 0, nb))
    return f16_bits(0.005 + 0.025 * u).reshape(n, k // 256)


def codebook(seed: int) -> np.ndarray:
    """fp16 bits [8][256][4], N(0,1)."""
    return f16_bits(_normals(key(seed, TAG_CODEBOOK), 0, 8 * 256 * 4)).reshape(8, 256, 4)


def activations(seed: int, m: int, k: int, stream: int = 0) -> np.ndarray:
    """bf16 bits [m][k], N(0,1).  `stream` selects an independent stream."""
    kk = key(seed, TAG_ACTIVATION ^ (stream << 12))
    return bf16_bits(_normals(kk, 0, m * k)).reshape(m, k)


def dense_weights(seed: int, n: int, k: int, std: float = 0.02, outlier_rate: float = 0.0,
                  outlier_gain: float = 8.0) -> np.ndarray:
    """bf16 bits [n][k]: unquantized weight rows, N(0, std^2) with a fraction
    `outlier_rate` of entries multiplied by `outlier_gain`."""
    z = _normals(key(seed, TAG_DENSE), 0, n * k) * std
    if outlier_rate > 0.0:
        u = _unit(draws(key(seed, TAG_DENSE | 1), 0, n * k))
        z = np.where(u < outlier_rate, z * outlier_gain, z)
    return bf16_bits(z).reshape(n, k)


def weight_rows_f32(seed: int, n: int, k: int, std: float = 1.0, row0: int = 0) -> np.ndarray:
    """fp32 [n][k]: N(0, std^2) rows row0 .. row0+n-1 of one seeded matrix
    with k columns (a stand-in for rotated weights)."""
    z = _normals(key(seed, TAG_DENSE | 2), row0 * k, n * k) * std
    return z.astype(np.float32).reshape(n, k)


def hessian_factor(seed: int, k: int, gamma: float = 0.5) -> np.ndarray:
    """fp32 [k][k]: block strictly upper factor U of a synthetic proxy Hessian
    H = (I + U)(I + U)^T (256-column blocks)."""
    z = _normals(key(seed, TAG_DENSE | 3), 0, k * k).reshape(k, k)
    bi = np.arange(k) // 256
    mask = bi[:, None] < bi[None, :]
    norm = np.sqrt(256.0 * np.maximum(bi, 1))[None, :]
    return np.where(mask, gamma * z / norm, 0.0).astype(np.float32)


def pack_bytes(n: int, k: int) -> int:
    """Bytes of codes + scales of one n x k weight (input sizing helper)."""
    return n * (k // 4) + 2 * n * (k // 256)


class Weight:
    """Host copy of one trellis-coded weight (inputs only)."""

    def __init__(self, seed: int, layer: int, op: int, n: int, k: int, cb: np.ndarray | None = None):
        self.seed, self.layer, self.op, self.n, self.k = seed, layer, op, n, k
        self.codes = codes(seed, layer, op, n, k)
        self.scales = scales(seed, layer, op, n, k)
        self.codebook = codebook(seed) if cb is None else cb


from .shapes import CONFIGS, StackShape, stack_shape  # noqa: E402,F401
