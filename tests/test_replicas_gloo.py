"""Multi-process host logic of `bench.py --gpus N` (replicas, max-over-ranks
timing) with two gloo ranks on the CPU."""
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


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        seconds = [1.0, 2.5][rank]
        value, t_max = bench.replica_throughput(100.0, seconds, world, device="cpu")
        q.put((rank, value, t_max))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, value, t_max in got:
        assert t_max == 2.5  # every rank agrees on the job's duration
        assert value == pytest.approx(200.0 / 2.5)  # all ranks' units over the slowest rank's time


def test_single_rank_is_plain_throughput():
    assert bench.replica_throughput(50.0, 2.0, 1) == (25.0, 2.0)
