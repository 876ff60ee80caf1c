"""Multi-process host logic of the bench on CPU (gloo, world size 2): each rank gets its own inputs,
and timings are reduced as the maximum over ranks.  The data path has no collective."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from block_sparse_attention_sum_b200.workloads import WORKLOADS

    w = WORKLOADS["tiny"]
    seed = bench.rank_seed(w, rank)
    q = torch.Generator().manual_seed(seed)
    first = torch.randn(4, generator=q)
    # rank r reports elapsed times [r + 1, 10 - r]; the slowest rank must win in each slot
    reduced = bench.max_over_ranks([rank + 1.0, 10.0 - rank], world)
    gathered = [None] * world
    dist.all_gather_object(gathered, (seed, first.tolist()))
    out[rank] = (reduced, gathered)
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_inputs_and_reduce_max():
    world = 2
    port = 29500 + (os.getpid() % 1000)
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        reduced, gathered = out[rank]
        assert reduced == [2.0, 10.0]
        seeds = [g[0] for g in gathered]
        assert len(set(seeds)) == world                 # distinct inputs per rank
        assert gathered[0][1] != gathered[1][1]
