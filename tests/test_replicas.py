"""Multi-rank host logic (world size 2, gloo backend on CPU): per-rank batches
and the max-over-ranks timing that bench.py uses for N > 1."""
import os

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_io_aware_70_b200.replicas import (SEED_STRIDE, job_throughput, max_over_ranks,
                                             rank_info, replica_workload)
from seeded_inputs import WORKLOADS, make_workload


def test_rank_info_parsing():
    assert rank_info({}) == rank_info({"WORLD_SIZE": "1", "RANK": "0"})
    r = rank_info({"WORLD_SIZE": "4", "RANK": "3", "LOCAL_RANK": "1"})
    assert (r.world_size, r.rank, r.local_rank) == (4, 3, 1)
    with pytest.raises(ValueError):
        rank_info({"WORLD_SIZE": "2", "RANK": "2"})


def test_job_throughput_is_weak_scaling():
    assert job_throughput(10.0, 4, 2.0) == 20.0


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = replica_workload(WORKLOADS["tiny"], rank)
        q, _, _ = make_workload(w)
        # each rank draws its own batch; timings reduce to the slowest rank
        t = max_over_ranks([1.0 + rank, 5.0 - rank])
        out[rank] = (w.seed, float(q.float().sum()), t)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    port = 29500 + os.getpid() % 1000
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn")
        r0, r1 = out[0], out[1]
    assert r1[0] - r0[0] == SEED_STRIDE          # distinct seeded batches
    assert r0[1] != r1[1]
    assert r0[2] == r1[2] == [2.0, 5.0]          # element-wise max over ranks
