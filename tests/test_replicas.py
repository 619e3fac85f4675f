"""Multi-GPU runs are independent replicas: the host-side timing logic of
bench.py (max over ranks, whole-job throughput) on world_size-2 gloo ranks
on the CPU. There is no collective on the data path to test."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_seconds = 1.0 + rank  # rank 1 is the slow one
        mx = bench.reduce_max_over_ranks(local_seconds, dist)
        value = bench.aggregate_throughput(8192 * 10, world, mx)
        q.put((rank, mx, value))
    finally:
        dist.destroy_process_group()


def test_replica_timing_takes_max_over_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, mx, value in got:
        assert mx == pytest.approx(2.0)
        assert value == pytest.approx(8192 * 10 * 2 / 2.0)


def test_single_process_reduce_is_identity():
    assert bench.reduce_max_over_ranks(3.5, None) == 3.5
    assert bench.aggregate_throughput(100, 1, 2.0) == 50.0
