"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The decode path shards with no exchange: each rank runs an independent replica
on its own seeded batch, and the only collective is the max over ranks of the
timings.  These tests run that reduction and the whole-job throughput formula
in two gloo processes, and check that the replicas draw different batches.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from paged_kv_cache_413_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (10 + r) ms for the whole run and (2 - r) ms per decode
        got = bench.max_over_ranks([10.0 + rank, 2.0 - rank], world)
        cfg = W.CONFIGS["tiny"]
        wl = W.make_workload(cfg, seed=cfg.seed + 1000 * rank) if rank else W.make_workload(cfg)
        out[rank] = (got, float(wl.query.float().sum()))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_seeds():
    world = 2
    mgr = mp.get_context("spawn").Manager()  # no fork of a threaded process
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0][0] == [11.0, 2.0] and out[1][0] == [11.0, 2.0]
    assert out[0][1] != out[1][1]  # each replica decodes its own batch


def test_whole_job_throughput_counts_every_replica():
    # 1 GB per step, 100 steps in 50 ms on each of 4 replicas -> 8 TB/s job-wide
    assert bench.whole_job_gbs(10**9, 4, 100, 50.0) == pytest.approx(8000.0)
    assert bench.max_over_ranks([3.0, 4.0], 1) == [3.0, 4.0]
