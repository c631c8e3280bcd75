"""Row-sharded layer stack over several GPUs (one process per GPU).

Every linear layer of the stack is split by output rows: rank r of P holds
rows [r N/P, (r+1) N/P) of each op's codes and scales (whole 16-row tiles),
the shared 16 KB codebook, and the full activation of every phase.  Each
phase then computes its RHT over the full input and the matmul of the local
rows only (tq_layer_phase on the local shards), and one all-gather of the
handed-on op's rows (bf16, rank order) rebuilds the next phase's full input.
The RHT mixes every 512-block of the input, so nothing smaller than the
whole handoff can feed the next phase: one exchange per phase is the least
this split needs.  The k, v and up outputs stay on their ranks.

Pages: "Pingala-8" landing page, "How it works" (the method) and
"Limitations" (one GPU in the pages' own runs); the split by output rows is
this library's reading of how the per-layer work divides, since every output
row depends on the whole input and on its own weight row only.

`run_stack` holds the sequencing (layer and phase order, per-(layer, phase)
seeds, the all-gather and its order) and takes the per-phase compute and the
gather as arguments, so the same logic drives the GPU path (`ShardedStack`:
libtq calls plus an NCCL all-gather) and the host-side tests.
"""
from __future__ import annotations

HANDOFF_OP = ("q", "o", "gate", "down")  # the op of each phase whose rows feed the next phase
PHASE_OPS = (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))


def row_shard(n: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [r0, r1) of an n-row op held by `rank`: equal, contiguous shards
    of whole 16-row tiles.  n must be a multiple of 16 * world."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    if n % (16 * world):
        raise ValueError(f"{n} rows do not split into {world} shards of whole 16-row tiles")
    per = n // world
    return rank * per, (rank + 1) * per


def run_stack(n_layers: int, h, phase_seed, compute_phase, gather):
    """The sharded stack's sequence.  For layer l and phase p: x is the full
    phase input; compute_phase(l, p, x, seed) returns this rank's rows of the
    handed-on op's bf16 output; gather(local) returns every rank's rows
    concatenated in rank order (the full next input).  Returns the final
    hidden state (full, on every rank)."""
    x = h
    for l in range(n_layers):
        for p in range(4):
            x = gather(compute_phase(l, p, x, phase_seed(l, p)))
    return x


class ShardedStack:
    """The row-sharded stack on this process's GPU.

    layers: one dict per layer of full DeviceWeights (q, k, v, o, gate, up,
    down) on this device; only the local rows are kept referenced (views of
    the same memory).  group: a torch.distributed process group (NCCL) of
    `world` ranks; rank = this process's rank in it."""

    def __init__(self, layers, rank: int, world: int, group=None, device=None):
        import torch

        from . import DeviceWeight, layer_struct, workspace
        self.rank, self.world, self.group = rank, world, group
        self.device = device if device is not None else layers[0]["q"].codes.device
        self.local = []
        for L in layers:
            loc = {}
            for op, w in L.items():
                r0, r1 = row_shard(w.n, world, rank)
                loc[op] = DeviceWeight(w.codes[r0:r1], w.scales[r0:r1], w.codebook, r1 - r0, w.k)
            self.local.append(loc)
        self.structs = [layer_struct(loc) for loc in self.local]
        self.n_layers = len(layers)
        self._ws = {}
        self._torch = torch
        self._workspace = workspace

    def _phase_ws(self, m):
        from . import tq_layer_phase_workspace
        if m not in self._ws:
            b = max(tq_layer_phase_workspace(s, p, m) for s in self.structs for p in range(4))
            self._ws[m] = self._workspace(b, self.device)
        return self._ws[m]

    def compute_phase(self, l: int, p: int, x, seed: int):
        """This rank's rows of phase p of layer l: bf16 handoff [m][n_local]."""
        from . import tq_layer_phase
        torch = self._torch
        m = x.shape[0]
        loc = self.local[l]
        ops = PHASE_OPS[p]
        y = torch.empty((m, sum(loc[o].n for o in ops)), dtype=torch.float32, device=self.device)
        hand = torch.empty((m, loc[HANDOFF_OP[p]].n), dtype=torch.int16, device=self.device)
        tq_layer_phase(self.structs[l], p, x.contiguous(), seed, y, hand, self._phase_ws(m))
        return hand

    def gather(self, local):
        """All-gather of every rank's handoff rows, in rank order (NCCL)."""
        torch = self._torch
        if self.world == 1:
            return local
        import torch.distributed as dist
        m, n = local.shape
        out = torch.empty((self.world, m, n), dtype=local.dtype, device=local.device)
        dist.all_gather_into_tensor(out, local.contiguous(), group=self.group)
        return out.permute(1, 0, 2).reshape(m, self.world * n)

    def forward(self, h, seed: int):
        """h: int16 (bf16 bits) [m][hidden] on this device; returns the final
        hidden state [m][hidden] on every rank."""
        from . import tq_stack_phase_seed
        return run_stack(self.n_layers, h, lambda l, p: tq_stack_phase_seed(seed, l, p), self.compute_phase,
                         self.gather)

