"""The multi-rank logic of bench.py on CPU: world-size-2 gloo process groups.

bench.py runs one replica per GPU (the path does not shard: each rank prefills its own
sequence); the ranks meet only to take the max of their times. These tests run that
reduction on two CPU processes, check the whole-job throughput, and check that the
reference arm runs on rank 0 alone."""
import os
import socket
import types

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    from datetime import timedelta

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        mine = [10.0, 12.5][rank]  # rank 1 is the slow one
        ms = bench.max_over_ranks(mine, world, "cpu")
        again = bench.max_over_ranks(3.0 + rank, world, "cpu")  # a second reduction, same order on every rank
        q.put((rank, ms, again, bench.job_throughput(1000.0, ms, world)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_on_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, again, thr in got:
        assert ms == 12.5 and again == 4.0
        assert thr == pytest.approx(2 * 1000.0 / 0.0125)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.0, 1, "cpu") == 7.0
    assert bench.job_throughput(131072, 250.0, 1) == pytest.approx(131072 / 0.25)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    # a rank other than 0 returns at once, before any oracle work
    def boom(*a, **k):
        raise AssertionError("rank 1 must not build the workload")

    monkeypatch.setattr(bench, "make_weights", boom)
    args = types.SimpleNamespace(steps=1, warmup=0)
    assert bench.run_reference(args, world=2, rank=1) == 0
