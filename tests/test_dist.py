"""The multi-process (N > 1) logic of bench.py on the CPU with two gloo ranks.

Each rank runs its own replica of the workload (weak scaling, no data-path
collective); the process group only provides barriers and the max over ranks
of the per-step time, which is what the reported value divides by.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, local = bench.dist_setup(world)
    assert (w, r, local) == (world, rank, rank)
    assert dist.get_backend() == "gloo"
    # each rank times a different amount of work; the job time is the slowest rank's
    ms = 1.0 + 2.5 * rank
    bench.barrier(w)
    got = bench.max_over_ranks(ms, w, torch.device("cpu"))
    results[rank] = got
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_barriers_on_gloo(world):
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        assert dict(results) == {r: 1.0 + 2.5 * (world - 1) for r in range(world)}


def test_single_process_needs_no_group():
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.dist_setup(1) == (1, 0, 0)
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    bench.barrier(1)
