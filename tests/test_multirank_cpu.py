"""The benchmark's multi-rank logic on CPU: two gloo ranks, each timing its
own replica; the reported step time is the max over ranks and the token
count the sum (weak scaling, no collective on the data path)."""

import os
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        t = bench.max_over_ranks(10.0 + rank)
        s = bench.sum_over_ranks(64.0)
        out[rank] = (r, w, lr, t, s, bench.rank_seed(0, rank))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timing_and_tokens():
    world, port = 2, 29517
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0][:3] == (0, 2, 0) and out[1][:3] == (1, 2, 1)
    assert out[0][3] == out[1][3] == 11.0          # max over ranks
    assert out[0][4] == out[1][4] == 128.0         # tokens summed over ranks
    assert out[0][5] != out[1][5]                  # each replica draws its own inputs


def test_single_process_reductions_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5 and bench.sum_over_ranks(2.0) == 2.0
