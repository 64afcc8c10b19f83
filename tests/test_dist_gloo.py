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
