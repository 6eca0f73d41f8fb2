"""The bench's multi-rank host logic on CPU ranks (gloo, world size 2).

The decode pass does not shard: N GPUs run N replicas, and the bench takes
the slowest rank's device time and the units all ranks processed.  Here two
gloo ranks on 127.0.0.1 exercise the barrier, the max over ranks and the
whole-job rate, and the reference arm leaves every rank but 0 idle.
"""
import datetime
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, queue):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 2.0 + rank            # rank 1 is the slower one
        slowest = bench.max_over_ranks(ms, world, device="cpu")
        bench.barrier(world)
        rate = bench.whole_job_rate(world, 1000, slowest)
        queue.put((rank, slowest, rate))
    finally:
        dist.destroy_process_group()


def test_two_ranks_report_the_slowest_rank_and_the_whole_job():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(queue.get(timeout=5) for _ in range(2))
    for rank, slowest, rate in got:
        assert slowest == 3.0
        # 2 ranks x 1000 units per step in 3 ms
        assert rate == pytest.approx(2 * 1000 / 3e-3)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(4.5, 1) == 4.5
    assert bench.whole_job_rate(1, 10, 2.0) == pytest.approx(5000.0)


def test_reference_arm_idles_on_other_ranks(capsys):
    sys.path.insert(0, ROOT)
    import argparse

    import bench

    args = argparse.Namespace(steps=3, warmup=3, gpus=2, impl="reference")
    assert bench.run_reference(args, world=2, rank=1) == 0
    assert capsys.readouterr().out == ""
