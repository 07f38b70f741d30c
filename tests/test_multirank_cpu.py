"""The N > 1 path of the benchmark on CPU: two ranks over gloo (127.0.0.1).
Each rank runs one independent replica; the job's time is the maximum over
the ranks, its throughput every replica's work over that time, and only
rank 0 prints (the reference arm's other ranks exit without work)."""
import argparse
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r "measured" (10 + r, 5 - r, 3 * r) ms
        got = bench.max_over_ranks([10.0 + rank, 5.0 - rank, 3.0 * rank], world, "cpu")
        ref = bench.run_reference(argparse.Namespace(steps=1, warmup=0), rank, world) if rank != 0 else "skip"
        q.put((rank, got, ref))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        rank, got, ref = q.get(timeout=120)
        out[rank] = (got, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    expect = [11.0, 5.0, 3.0]  # max over ranks, per value
    assert out[0][0] == expect and out[1][0] == expect
    assert out[1][1] is None   # the reference arm does nothing on rank 1


def test_whole_job_value_counts_every_replica():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_tops(1, 10.1e12, 5, 4000.0)
    two = bench.whole_job_tops(2, 10.1e12, 5, 4000.0)
    assert two == pytest.approx(2 * one)
    assert one == pytest.approx(10.1 * 5 / 4.0)
