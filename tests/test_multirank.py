"""Multi-rank plumbing of bench.py on CPU: two gloo ranks (world size 2).

The forward shards over independent (batch, kv head) chains, so the benchmark's only
collectives are the timing barrier and a max / sum over ranks; these run here on gloo.
"""
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


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        w, r, l = bench.dist_env()
        assert (w, r, l) == (world, rank, rank)
        bench.barrier(world)
        mx = bench.max_over_ranks(float(rank + 1) * 1.5, world, "cpu")
        sm = bench.sum_over_ranks(float(rank + 1), world, "cpu")
        bench.barrier(world)
        results[rank] = (mx, sm)
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_collectives():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        assert results[r] == (3.0, 3.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import argparse
    import bench
    from compressive_memory_long_b200 import workloads as wl
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    called = []
    monkeypatch.setattr(bench, "oracle_sample", lambda *a, **k: called.append(1))
    args = argparse.Namespace(steps=2, warmup=3, gpus=2)
    assert bench.run_reference(args, wl.WORKLOADS["fp32_linear_small"]) == 0
    assert called == []


def test_single_rank_helpers_are_identity():
    import bench
    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5
    assert bench.sum_over_ranks(2.5, 1, "cpu") == 2.5
    bench.barrier(1)
