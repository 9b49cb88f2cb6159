"""The benchmark's multi-rank logic on CPU: two gloo ranks, max-over-ranks timing,
weak-scaling throughput, and the reference arm's rank-0-only rule."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, _ = bench.dist_setup()
        assert (w, r) == (world, rank)
        step = 0.05 + 0.01 * rank              # rank 1 is the slowest
        bench.barrier(world)
        m = bench.max_over_ranks(step, world)
        v = bench.whole_job_value(1e12, m, world)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_step_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, v in got:
        assert m == pytest.approx(0.06)
        assert v == pytest.approx(2 * 1e12 / 0.06 / 1e12)


def test_reference_arm_runs_only_on_rank_zero(monkeypatch):
    class A:
        workload, topk, steps, warmup, gpus = "tiny", 0.5, 1, 1, 2

    called = []
    monkeypatch.setattr(bench.W, "make_qkv", lambda wl: called.append(1))
    assert bench.run_reference(A(), world=2, rank=1) == 0
    assert not called


def test_single_rank_helpers():
    assert bench.max_over_ranks(0.123, 1) == 0.123
    assert bench.whole_job_value(2e12, 0.5, 1) == pytest.approx(4.0)
