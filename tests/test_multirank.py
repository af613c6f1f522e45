"""The N > 1 path of bench.py on CPU: world_size-2 gloo ranks. Each rank is an independent
replica (the path shards into independent sequences, no collective on the data path); the
only collectives are the barrier and the max-over-ranks reduction of the timings."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world)     # rank 1 is the slow one
        val = bench.replica_value(32 * 100, world, ms)            # 100 steps of 32 tokens per rank
        out[rank] = (ms, val)
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_take_the_slowest_time():
    world = 2
    out = mp.Manager().dict()
    mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][1] == pytest.approx(32 * 100 * 2 / 0.015)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.replica_value(320, 1, 10.0) == pytest.approx(32000.0)
