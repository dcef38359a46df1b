"""The multi-rank bench path on CPU ranks (gloo, world size 2): the step time is the max over
ranks, every rank draws its own sequences (weak scaling), and ranks agree on the result."""
from __future__ import annotations

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
    try:
        import bench
        from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs
        t = bench.max_over_ranks(10.0 + rank, world)
        w = WORKLOADS["decode_b8_ctx128k_ragged"].scaled(batch=2, max_seq_len=256, min_seq_len=64, n_q_heads=8,
                                                         n_kv_heads=2, n_idx_k_heads=2, hot_blocks=1,
                                                         block_size=64, top_k=2)
        x = make_inputs(w, seed=bench.rank_seed(w, rank))
        digest = torch.tensor([float(x["k_idx"].float().sum()), float(x["seq_lens"].sum())])
        all_d = [torch.zeros(2) for _ in range(world)]
        dist.all_gather(all_d, digest)
        bench.barrier(world)
        out[rank] = (t, [d.tolist() for d in all_d])
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_shards():
    world = 2
    port = 29500 + (os.getpid() % 1000)
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    t0, d0 = out[0]
    t1, d1 = out[1]
    assert t0 == t1 == 11.0               # both ranks report the slowest rank's time
    assert d0 == d1                        # ranks agree on what everyone drew
    assert d0[0] != d0[1]                  # and each rank drew different sequences
