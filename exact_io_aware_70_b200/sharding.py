"""How the hot path is split over several GPUs (one process per GPU).

Two splits, both from the structure of the method:

* Prefill: every (batch, head) pair is an independent attention problem, so a
  batch of B x H heads is cut into contiguous ranges of the flattened (b, h)
  index, one range per rank (``head_range``). A rank runs ``attn_fwd`` on its
  range as one dense [1, H_r, N, d] view; no data crosses GPUs.
* Decode: with one query row the parallelism is in the keys. The pages split
  the KV sequence across thread blocks and merge the per-chunk partials with
  the max-and-sum trick ("Describe Flash Attention at a high level"
  (mantramindai), "Follow-up questions to expect", last question); here the
  same split is carried one level up. Rank r holds a contiguous shard of the
  keys (``kv_range``), computes its S chunk partials (O_c, lse_c) with
  ``attn_decode_partials``, the ranks all-gather the partials
  (B x H x S x (d + 1) fp32 per rank, 264 KB at 16 x 32 heads, d = 128,
  S = 64), and every rank merges the R x S chunks with
  ``attn_lse_merge_gathered``. The merge does not depend on where the chunk
  boundaries fall, so the result equals the single-GPU one up to rounding.

The orchestration (``kv_split_decode``) takes the per-shard partial step and
the merge as functions, so the same rank logic runs the CUDA library on GPUs
(NCCL) and, in the tests, the CPU oracle on gloo ranks.
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


def balanced_range(n: int, rank: int, world: int) -> tuple[int, int]:
    """[lo, hi) of rank's share of n items cut into `world` contiguous pieces
    whose sizes differ by at most one (the first n % world pieces are longer)."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError(f"bad split of {n} items: rank {rank} of {world}")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def head_range(B: int, H: int, rank: int, world: int) -> tuple[int, int]:
    """Rank's contiguous range of the flattened (b, h) index of a [B, H, N, d] batch."""
    return balanced_range(B * H, rank, world)


def kv_range(Nkv: int, rank: int, world: int) -> tuple[int, int]:
    """Rank's contiguous shard [lo, hi) of the key sequence for the split decode."""
    return balanced_range(Nkv, rank, world)


def gather_partials(o_part, lse_part, group=None):
    """All-gather every rank's partials: [B, H, S, d] and [B, H, S] in, the
    stacked [R, B, H, S, d] and [R, B, H, S] out, rank r at index r (the layout
    ``attn_lse_merge_gathered`` reads). Without a process group R = 1."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return o_part.unsqueeze(0), lse_part.unsqueeze(0)
    R = dist.get_world_size(group)
    o_part, lse_part = o_part.contiguous(), lse_part.contiguous()
    og = torch.empty((R,) + tuple(o_part.shape), dtype=o_part.dtype, device=o_part.device)
    lg = torch.empty((R,) + tuple(lse_part.shape), dtype=lse_part.dtype, device=lse_part.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(og, o_part, group=group)
        dist.all_gather_into_tensor(lg, lse_part, group=group)
    else:
        dist.all_gather(list(og.unbind(0)), o_part, group=group)
        dist.all_gather(list(lg.unbind(0)), lse_part, group=group)
    return og, lg


def kv_split_decode(q, k_shard, v_shard, scale: float, splits: int, partials, merge, group=None):
    """One split-KV decode step across the ranks of `group`.

    q [B, H, 1, d] is the same on every rank; k_shard, v_shard [B, H, n_r, d]
    are this rank's keys (``kv_range``). ``partials(q, k, v, scale, S)`` returns
    this rank's (o_part [B, H, S, d], lse_part [B, H, S]); ``merge(og, lg)``
    merges the gathered [R, ...] partials into (o, lse). Every rank returns the
    merged result."""
    o_p, l_p = partials(q, k_shard, v_shard, scale, splits)
    og, lg = gather_partials(o_p, l_p, group)
    return merge(og, lg)


SEED_STRIDE = 1000


def shard_seed(seed: int, rank: int) -> int:
    """Seed of rank's slice of a workload that grows with the number of GPUs
    (its own batch entries for the prefill, its own key shard for the decode)."""
    return seed + SEED_STRIDE * rank


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
