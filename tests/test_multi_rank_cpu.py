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


def _reference_worker(rank, world, port, results):
    """A rank of `bench.py --impl reference --gpus 2`: the process group comes from the bench's
    own setup (gloo without a device); rank 0 alone times the oracle and prints its line."""
    import contextlib
    import io
    import types

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    from gated_linear_attention_liger_b200 import inputs
    bench.PREFILL = inputs.small("multi_rank_reference", B=1, Hq=2, Hkv=1, T=128, d=64, seed=4)
    sample = bench.oracle_prefill_sample
    bench.oracle_prefill_sample = lambda target_s: sample(0.1)
    args = types.SimpleNamespace(gpus=world, steps=1, warmup=0)
    w, r, _ = bench.dist_setup(args)
    out = io.StringIO()
    try:
        with contextlib.redirect_stdout(out):
            bench.run_reference(args, w, r)
    finally:
        dist.destroy_process_group()
    results[rank] = (w, r, out.getvalue())


def test_reference_arm_under_two_ranks():
    import json
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_reference_worker, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
            assert p.exitcode == 0
        assert results[0][:2] == (2, 0) and results[1][:2] == (2, 1)
        assert results[1][2] == ""
        lines = results[0][2].strip().splitlines()
        assert len(lines) == 1
        line = json.loads(lines[0])
        assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
