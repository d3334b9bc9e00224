"""Host logic of the multi-GPU benchmark on CPU: world-size-2 gloo ranks.

Sequences are independent, so each rank runs its own copy of the workload
(weak scaling) and the only cross-rank steps are a barrier and the max of the
per-rank times.  No GPU is touched."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        ms = 3.0 + rank          # rank 1 is the slow one
        worst = bench.max_over_ranks(ms, world, torch.device("cpu"))
        results[rank] = (worst, bench.weak_scaling_value(16384, world, worst))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        assert results[0][0] == pytest.approx(4.0) and results[1][0] == pytest.approx(4.0)
        assert results[0][1] == pytest.approx(2 * 16384 / 4e-3)
