"""The benchmark's multi-rank plumbing on CPU: two gloo ranks reduce their
device times to the slowest one, as the NCCL ranks of `bench.py --gpus N` do
(replicas: each rank runs its own copy of the workload, no data exchange)."""

from __future__ import annotations

import datetime
import os
import socket

import pytest

torch = pytest.importorskip("torch")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    got = bench.reduce_max(1.5 + rank, world, "cpu")
    dist.barrier()
    dist.destroy_process_group()
    queue.put((rank, got))


def test_two_ranks_take_the_slowest_time():
    ctx = torch.multiprocessing.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(queue.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results == {0: 2.5, 1: 2.5}


def test_single_rank_is_its_own_value():
    import bench
    assert bench.reduce_max(3.25, 1, "cpu") == 3.25
