"""Host logic of the multi-GPU benchmark on CPU ranks (gloo, world size 2).

The decode workload shards by sequence (weak scaling): every rank draws its own
batch from a rank-specific seed, runs with no data-path collective, and the
job's time is the slowest rank's. These checks run the same helpers bench.py
uses under torchrun, on two CPU processes.
"""
import datetime
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from long_context_indexer_b200.workloads import CONFIGS, generate

        cfg = CONFIGS["tiny"]
        w = generate(cfg, seed=cfg.seed + bench.shard_seed_offset(rank))
        local = [10.0 + 4.0 * rank, 3.0 - rank]
        total = bench.reduce_max_ms(local, torch.device("cpu"), world)
        value = bench.job_throughput(world, cfg.B * cfg.S, 50, total[0])
        digest = float(w["q"].double().sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, digest)
        out[rank] = (total, value, gathered)
    finally:
        dist.destroy_process_group()


def test_weak_scaling_reduction_two_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        total, value, digests = out[rank]
        assert total == [14.0, 3.0]                      # max over ranks, per timing
        assert value == pytest.approx(2 * 256 * 50 / 0.014)
        assert digests[0] != digests[1]                  # each rank draws its own batch


def _cp_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from long_context_indexer_b200 import cp
        ranges = cp.shard_ranges(8193, world)
        lo, hi = ranges[rank]
        # each rank contributes its (scores, ids) lists; every rank must see all
        # of them, in rank order
        ids = torch.arange(lo, lo + 6, dtype=torch.int32).reshape(1, 2, 3)
        scores = torch.full((1, 2, 3), float(rank), dtype=torch.float32)
        g_ids = cp.all_gather(ids)
        g_scores = cp.all_gather(scores)
        out[rank] = (ranges, g_ids.tolist(), g_scores.tolist())
    finally:
        dist.destroy_process_group()


def test_context_parallel_exchange_two_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_cp_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    ranges = out[0][0]
    assert ranges == [(0, 4097), (4097, 8193)]       # contiguous, covering, near-equal
    for rank in range(world):
        _, g_ids, g_scores = out[rank]
        assert g_ids == out[0][1]                     # the same on every rank
        for r, (lo, _) in enumerate(ranges):
            assert g_ids[r] == torch.arange(lo, lo + 6).reshape(1, 2, 3).tolist()
            assert g_scores[r] == [[[float(r)] * 3] * 2]


def test_shard_ranges_cover_without_overlap():
    from long_context_indexer_b200 import cp
    for nb in (1, 7, 8192, 8193):
        for world in (1, 2, 3, 8):
            rs = cp.shard_ranges(nb, world)
            assert rs[0][0] == 0 and rs[-1][1] == nb and len(rs) == world
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            sizes = [hi - lo for lo, hi in rs]
            assert max(sizes) - min(sizes) <= 1
