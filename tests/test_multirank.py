"""The multi-GPU bench path (replicas: barrier, max-over-ranks device time,
whole-job throughput), exercised as two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, ms_by_rank, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        ms = bench.max_over_ranks(ms_by_rank[rank], dist, world, device="cpu")
        v = bench.job_throughput(84, 10, world, ms)
        q.put((rank, ms, v))
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank():
    world, port = 2, _free_port()
    ms_by_rank = [12.5, 20.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, ms_by_rank, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, v in got:
        assert ms == 20.0                       # every rank sees the max
        assert v == pytest.approx(84 * 10 * 2 / 0.020)  # units of all ranks / max time


def test_single_rank_is_unchanged():
    assert bench.max_over_ranks(3.0, None, 1) == 3.0
    assert bench.job_throughput(42, 5, 1, 1000.0) == pytest.approx(210.0)
