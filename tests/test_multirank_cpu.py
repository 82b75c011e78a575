"""The multi-rank host logic of bench.py on CPU: two gloo ranks."""
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
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from indexed_sparse_attention_kv_b200 import inputs as I

        w = I.workload("decode_128k")
        mine = [10.0 + rank, 20.0 - rank]                 # rank 1 slower on the first value
        got = bench.max_over_ranks(mine, world)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(w, rank))
        out[rank] = (got, seeds)
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction():
    world = 2
    mgr = mp.get_context("spawn").Manager()   # no fork of a threaded process
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        got, seeds = out[r]
        assert got == [11.0, 20.0]                     # max over ranks, elementwise
        assert len(set(seeds)) == world                # every rank decodes its own sequences


def test_weak_value():
    import bench
    assert bench.weak_value(1, 50, 5000.0) == pytest.approx(10.0)
    assert bench.weak_value(4, 50, 5000.0) == pytest.approx(40.0)
