"""The row-sharded stack's host logic on CPU: two gloo ranks, each computing
its own rows of every phase with the oracle, all-gather the handoffs in rank
order through decode_matmul_b200.sharded.run_stack; the result must be the
unsharded oracle stack bit for bit (every output row depends only on the full
input and its own weight row, so a correct split and gather order change
nothing)."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
import tqsynth
from decode_matmul_b200 import sharded

SHAPE = tqsynth.StackShape("shard-test", 2, 512, 1024, 512, 1536)
SEED = 77


def _weights():
    cb = tqsynth.codebook(5)
    return [{op: (tqsynth.codes(5, l, i, n, k), tqsynth.scales(5, l, i, n, k), cb, n, k)
             for i, (op, n, k) in enumerate(SHAPE.ops())} for l in range(SHAPE.layers)]


def _rank(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        layers = _weights()
        m = 2
        h = tqsynth.activations(9, m, SHAPE.hidden)

        def compute(l, p, x, seed):
            local = {}
            for op, (c, s, cb, n, k) in layers[l].items():
                r0, r1 = sharded.row_shard(n, world, rank)
                local[op] = (c[r0:r1], s[r0:r1], cb, r1 - r0, k)
            _, hand = oracle.stack_phase(p, x, m, local, seed)
            return hand

        def gather(local):
            # bf16 bit patterns, widened to int32 for gloo
            t = torch.from_numpy(local.astype(np.int32))
            parts = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(parts, t)
            return np.concatenate([x.numpy().astype(np.uint16) for x in parts], axis=1)

        out = sharded.run_stack(SHAPE.layers, h, lambda l, p: oracle.stack_phase_seed(SEED, l, p), compute, gather)
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_row_shard():
    assert sharded.row_shard(4096, 4, 0) == (0, 1024)
    assert sharded.row_shard(4096, 4, 3) == (3072, 4096)
    assert sharded.row_shard(9728, 8, 7) == (8512, 9728)
    for bad in [(1000, 2, 0), (4096, 3, 0)]:
        with pytest.raises(ValueError):
            sharded.row_shard(*bad)
    with pytest.raises(ValueError):
        sharded.row_shard(4096, 2, 2)


def test_two_gloo_ranks_reproduce_the_unsharded_stack():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want, _ = oracle.layer_stack(_weights(), tqsynth.activations(9, 2, SHAPE.hidden), 2, SEED)
    for r in range(2):
        assert np.array_equal(got[r], want), r


@pytest.mark.gpu
def test_sharded_phases_on_one_gpu_match_the_unsharded_phase():
    # two row shards computed one after the other on one GPU (no rank waits
    # on another), gathered in rank order, against the whole layer's phase
    # on the same input; a shard's unit split differs, so fp32 sums may
    # associate differently: the bf16 handoffs agree within one bf16 step
    import torch

    import decode_matmul_b200 as tq
    dev = torch.device("cuda", 0)
    cbd = torch.from_numpy(tqsynth.codebook(5).view(np.int16)).to(dev)
    layers = [{op: tq.DeviceWeight.from_host(tqsynth.codes(5, l, i, n, k), tqsynth.scales(5, l, i, n, k), cbd, n, k,
                                             device=dev)
               for i, (op, n, k) in enumerate(SHAPE.ops())} for l in range(SHAPE.layers)]
    shards = [sharded.ShardedStack(layers, r, 2) for r in range(2)]
    full = [tq.layer_struct(L) for L in layers]
    for m in (1, 3):
        ws = tq.workspace(max(tq.tq_layer_phase_workspace(s, p, m) for s in full for p in range(4)), dev)
        x = torch.from_numpy(tqsynth.activations(9, m, SHAPE.hidden).view(np.int16)).to(dev)
        for l in range(SHAPE.layers):
            for p in range(4):
                seed = tq.tq_stack_phase_seed(SEED, l, p)
                got = torch.cat([s.compute_phase(l, p, x, seed) for s in shards], dim=1)
                n_all = sum(layers[l][o].n for o in sharded.PHASE_OPS[p])
                y = torch.empty((m, n_all), dtype=torch.float32, device=dev)
                want = torch.empty_like(got)
                tq.tq_layer_phase(full[l], p, x, seed, y, want, ws)
                g = tqsynth.bf16_to_f64(got.cpu().numpy().view(np.uint16))
                w = tqsynth.bf16_to_f64(want.cpu().numpy().view(np.uint16))
                assert oracle.rel_err(g, w) < 1e-2, (m, l, p)
                x = got
