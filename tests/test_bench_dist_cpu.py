"""bench.py's multi-process plumbing on CPU (gloo, world size 2): max-over-ranks
timing and the weak-scaling aggregate, the same calls the NCCL run makes."""

from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, w, local = bench.dist_env()
    t_mine = 0.010 * (rank + 1)          # rank 1 is the slow one
    t_max = bench.reduce_max(t_mine, device="cpu")
    bench.barrier()
    out[rank] = (r, w, local, t_max, bench.weak_scaling_value(1.0e9, w, t_max))
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling():
    world = 2
    mgr = mp.get_context("spawn").Manager()  # no fork of this multi-threaded process
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        r, w, local, t_max, value = out[rank]
        assert (r, w, local) == (rank, world, rank)
        assert t_max == pytest.approx(0.020)
        assert value == pytest.approx(2 * 1.0e9 / 0.020)


def test_single_process_identity():
    import bench
    assert bench.reduce_max(1.5) == 1.5
    assert bench.weak_scaling_value(10.0, 1, 2.0) == 5.0
