"""Host-side plumbing for running the hot path on several GPUs as replicas.

The path has no exchange step: every (batch, head) work unit is independent,
so N GPUs run N independent replicas, each on its own seeded batch, and the
job's throughput is the work of all ranks divided by the slowest rank's time
(weak scaling). This module holds that logic so it can be tested with the
gloo backend on CPU; the kernels themselves never see it.
"""
from __future__ import annotations

import dataclasses
import os


@dataclasses.dataclass(frozen=True)
class RankInfo:
    world_size: int
    rank: int
    local_rank: int


def rank_info(env=None) -> RankInfo:
    """RANK / LOCAL_RANK / WORLD_SIZE as set by torch.distributed.run (defaults: one process)."""
    env = os.environ if env is None else env
    ws = int(env.get("WORLD_SIZE", "1"))
    rank = int(env.get("RANK", "0"))
    local = int(env.get("LOCAL_RANK", str(rank)))
    if ws < 1 or not 0 <= rank < ws:
        raise ValueError(f"bad rank {rank} for world size {ws}")
    return RankInfo(ws, rank, local)


SEED_STRIDE = 1000


def replica_workload(workload, rank: int):
    """The rank's own batch: the same shapes, seed offset by SEED_STRIDE * rank."""
    return dataclasses.replace(workload, seed=workload.seed + SEED_STRIDE * rank)


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(units_per_rank: float, world_size: int, seconds_max_over_ranks: float) -> float:
    """Whole-job rate: work of all ranks over the slowest rank's time."""
    return units_per_rank * world_size / seconds_max_over_ranks
