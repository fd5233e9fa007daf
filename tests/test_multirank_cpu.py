"""The bench's multi-rank plumbing on CPU: two gloo ranks, max over ranks of
the timed region and the barrier the timed region is bracketed by."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, lr = bench.dist_env()
    assert (r, w, lr) == (rank, world, rank)
    bench.dist_init(w, "gloo")
    bench.barrier(w)
    m = bench.reduce_max(10.0 * (rank + 1), w)
    out[rank] = m
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert dict(out) == {0: 20.0, 1: 20.0}


def test_single_rank_is_identity():
    assert bench.reduce_max(3.5, 1) == 3.5
