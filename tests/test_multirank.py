"""The multi-process side of bench.py on CPU: two gloo ranks take the
barrier and agree on the slowest rank's time (the job's time), as the GPU
ranks do over NCCL."""
from __future__ import annotations

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        t = bench.allreduce_max(10.0 + rank * 2.5, world)
        q.put((rank, t))
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(world))
    assert got == {0: 12.5, 1: 12.5}  # rank 1 is the slower one


def test_single_rank_is_identity():
    assert bench.allreduce_max(3.25, 1) == 3.25
