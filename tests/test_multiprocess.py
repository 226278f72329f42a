"""Multi-rank host logic of the benchmark on CPU (gloo, two ranks).

The pass shards by sequence with no data-path collective: each rank owns a contiguous block
of sequences and the only cross-rank operation is the max of the step time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}")
    try:
        mine = bench.shard_sequences(8, rank, world)
        t = bench.reduce_max(1.5 + rank, dist)
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        out[rank] = (mine, t, gathered)
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_reduce():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    (m0, t0, g0), (m1, t1, _) = out[0], out[1]
    assert m0 == [0, 1, 2, 3] and m1 == [4, 5, 6, 7]
    assert sorted(g0[0] + g0[1]) == list(range(8))          # every sequence exactly once
    assert t0 == t1 == 2.5                                   # max over ranks


def test_single_rank_is_identity():
    import bench
    assert bench.shard_sequences(4, 0, 1) == [0, 1, 2, 3]
    assert bench.reduce_max(3.25, None) == 3.25
