"""Rank plumbing of bench.py with world size 2 on the CPU (gloo).

The path has no collective on its data: replicas only.  What multi-process
runs share is the barrier around the timed region and the max over ranks of
the device time, which these tests exercise without a GPU.
"""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    ws, r, local = bench.dist_env()
    assert (ws, r, local) == (world, rank, rank)
    bench.init_dist(ws, "gloo")
    bench.barrier(ws)
    t = bench.max_over_ranks(1.5 + rank, ws, "cpu")
    out[rank] = t
    bench.barrier(ws)
    dist.destroy_process_group()


def test_max_over_ranks_world_size_2():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0] == out[1] == 2.5


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0, 1, "cpu") == 3.0
    bench.barrier(1)
