"""The multi-GPU bench path on CPU: two gloo ranks run the replica helpers.

Every step of the path is per head, so N ranks run N independent problems of
the same shape (weak scaling) and exchange nothing but their timings: the
job's step time is the slowest rank's, and the job's throughput is all ranks'
work over that time.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from synthetic import CONFIGS, make_qkv


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = bench.rank_workload(CONFIGS["tiny_topk"], rank)
        x = make_qkv(wl)
        times = [10.0 + rank, 5.0 - rank]                     # per-rank fake timings (ms)
        mx = bench.max_over_ranks(times, dist, "cpu")
        digest = float(x["q"].astype(np.float64).sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, (wl.config_id, x["q"].shape, digest))
        out[rank] = (mx, gathered)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replicas_and_max_timing():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    for r in range(world):
        mx, gathered = out[r]
        assert mx == [11.0, 5.0]                               # slowest rank per entry
        ids = [g[0] for g in gathered]
        assert len(set(ids)) == world                          # each rank: its own problem
        assert len({g[1] for g in gathered}) == 1              # of the same shape
        assert gathered[0][2] != gathered[1][2]                # with different data


def test_single_rank_helpers_and_aggregate():
    assert bench.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]
    # 4 ranks, each 8.582 TFLOP per step, slowest rank 10 ms -> 3432.8 TFLOP/s
    assert abs(bench.aggregate_tflops(4, 8.582e12, 10.0) - 3432.8) < 1e-6
