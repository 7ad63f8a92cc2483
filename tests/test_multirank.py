"""The multi-rank benchmark plumbing on CPU with the gloo backend (world size 2):
the reported time is the slowest rank's, every rank draws an independent
batch, and the aggregate counts the units of all ranks.  No kernel runs."""
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


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = [0.25, 0.75][rank]
        slowest = bench.max_over_ranks(elapsed, world)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(1002, rank))
        bench.barrier(world)
        results[rank] = (slowest, seeds)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_time():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.start_processes(_worker, args=(world, port, results), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(results)
    assert res[0][0] == res[1][0] == 0.75
    seeds = res[0][1]
    assert len(set(seeds)) == world                  # independent batches per rank
    assert bench.aggregate(1.0e9, world, 0.75) == pytest.approx(2.0e9 / 0.75)
