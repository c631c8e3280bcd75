"""The N > 1 path of bench.py (independent replicas) on CPU: two gloo ranks
run the same seeded workload and the timing is the maximum over ranks."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import tqsynth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # every replica builds the same seeded inputs
        h = tqsynth.activations(0, 1, 2560)
        digest = torch.tensor([float(np.frombuffer(h.tobytes(), dtype=np.uint16).astype(np.int64).sum())],
                              dtype=torch.float64)
        allh = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(allh, digest)
        ms = 1.0 + 0.5 * rank  # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        out.put((rank, [float(t.item()) for t in allh], ms_max,
                 bench.replica_throughput(1, world, 20, ms_max)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas_time_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, digests, ms_max, value in res:
        assert digests[0] == digests[1]  # identical seeded inputs on both replicas
        assert ms_max == 1.5
        assert value == pytest.approx(2 / 1.5e-3)


def test_single_process_paths():
    assert bench.max_over_ranks(3.25, None, None) == 3.25
    assert bench.replica_throughput(16, 1, 10, 4.0) == pytest.approx(16 / 4e-3)
