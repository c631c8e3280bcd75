"""Workload shapes: the synthetic stand-ins for the pages' models.

The pages measure Qwen3-4B, Llama-3.1-8B and a 27B-class model; no trained
weights are available, so these are random trellis-coded layers with the
models' linear-layer shapes (hidden size, attention projection widths and
MLP width).  A layer is q, k, v, o, gate, up, down; n = output features,
k = input features.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class StackShape:
    name: str
    layers: int
    hidden: int
    q_dim: int
    kv_dim: int
    inter: int

    def ops(self):
        """(op name, n, k) for the seven linear layers of one layer."""
        h, q, kv, i = self.hidden, self.q_dim, self.kv_dim, self.inter
        return [("q", q, h), ("k", kv, h), ("v", kv, h), ("o", h, q),
                ("gate", i, h), ("up", i, h), ("down", h, i)]

    def weights_per_layer(self) -> int:
        return sum(n * k for _, n, k in self.ops())

    def packed_bytes_per_layer(self) -> int:
        return sum(n * (k // 4) + 2 * n * (k // 256) for _, n, k in self.ops())

    def packed_bytes(self) -> int:
        return self.layers * self.packed_bytes_per_layer()


QWEN3_4B = StackShape("qwen3-4b-shaped", 36, 2560, 4096, 1024, 9728)
LLAMA31_8B = StackShape("llama-3.1-8b-shaped", 32, 4096, 4096, 1024, 14336)
CLASS_27B = StackShape("27b-class", 64, 5120, 6144, 1024, 17408)

STACKS = {s.name: s for s in (QWEN3_4B, LLAMA31_8B, CLASS_27B)}


def stack_shape(name: str, layers: int | None = None) -> StackShape:
    s = STACKS[name]
    if layers is not None:
        s = StackShape(s.name, layers, s.hidden, s.q_dim, s.kv_dim, s.inter)
    return s


# The five workloads: one single layer and four stack configurations.
CONFIGS = {
    "single-1024": dict(kind="linear", n=1024, k=1024, m=1, seed=0),
    "qwen3-4b-m1": dict(kind="stack", stack="qwen3-4b-shaped", m=1, seed=0),
    "qwen3-4b-m512": dict(kind="stack", stack="qwen3-4b-shaped", m=512, seed=0),
    "llama-8b-sweep": dict(kind="stack", stack="llama-3.1-8b-shaped", m=(1, 4, 8, 16), seed=0),
    "27b-sweep": dict(kind="stack", stack="27b-class", m=(1, 8, 32, 64), seed=0),
}
