"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (127.0.0.1) check the
max-over-ranks timing reduction and the whole-job value, and the reference arm
does its work on rank 0 only.  No GPU is used."""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        worst = bench.max_over_ranks(10.0 + rank, world)     # per-rank total ms
        bench.barrier(world)
        v = bench.job_value(world, steps=4, flops_per_step=2e12, total_ms_max=worst)
        q.put((rank, worst, v))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_the_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get() for _ in range(world))
    for rank, worst, v in got:
        assert worst == 11.0                       # the slower rank's time, on every rank
        # 2 ranks x 4 steps x 2 TFLOP in 11 ms of the slowest rank
        assert v == pytest.approx(2 * 4 * 2e12 / 11.0 / 1e9)


def test_job_value_single_rank_is_plain_throughput():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_value(1, 10, 1.6e12, 20.0) == pytest.approx(800.0)
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        steps, warmup, gpus = 1, 3, 2
    bench.run_reference(Args, world=2, rank=1)     # returns at once, prints nothing
    assert capsys.readouterr().out == ""
