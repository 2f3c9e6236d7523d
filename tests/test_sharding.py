"""Multi-rank logic of the split path on CPU (gloo, world size 2 and 3).

The decode split across GPUs (each rank holds a contiguous shard of the keys,
computes per-chunk partials, the ranks all-gather them and every rank merges
them with the max-and-sum trick -- "Describe Flash Attention at a high level"
(mantramindai), "Follow-up questions to expect", last question) is run here
with the fp64 oracle as the compute step, so the rank logic itself is checked:
the shards must cover every key exactly once, the gather must keep the ranks'
partials apart, and the merged result must equal the unsplit oracle to 1e-12.
The prefill split (heads partitioned over ranks) is checked the same way.
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_io_aware_70_b200.sharding import (SEED_STRIDE, balanced_range, gather_partials,
                                             head_range, job_throughput, kv_range,
                                             kv_split_decode, max_over_ranks, rank_info,
                                             shard_seed)


def test_rank_info_parsing():
    assert rank_info({}) == rank_info({"WORLD_SIZE": "1", "RANK": "0"})
    r = rank_info({"WORLD_SIZE": "4", "RANK": "3", "LOCAL_RANK": "1"})
    assert (r.world_size, r.rank, r.local_rank) == (4, 3, 1)
    with pytest.raises(ValueError):
        rank_info({"WORLD_SIZE": "2", "RANK": "2"})


@pytest.mark.parametrize("n,world", [(0, 1), (1, 3), (7, 2), (32768, 8), (100, 7), (5, 5)])
def test_balanced_ranges_cover_every_item_once(n, world):
    ranges = [balanced_range(n, r, world) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == n
    for (a, b), (c, _) in zip(ranges, ranges[1:]):
        assert b == c                                   # contiguous, no gap, no overlap
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == n
    assert head_range(2, n, 0, world) == balanced_range(2 * n, 0, world)
    assert kv_range(n, world - 1, world) == ranges[-1]


def test_job_throughput_and_seeds():
    assert job_throughput(10.0, 4, 2.0) == 20.0
    assert shard_seed(4, 3) - shard_seed(4, 0) == 3 * SEED_STRIDE


def test_gather_without_process_group_is_one_rank():
    o, lse = torch.zeros(2, 3, 4, 8), torch.zeros(2, 3, 4)
    og, lg = gather_partials(o, lse)
    assert og.shape == (1, 2, 3, 4, 8) and lg.shape == (1, 2, 3, 4)


# ---------------------------------------------------------------- gloo ranks --
def _oracle_partials(q, k, v, scale, S):
    """Per-chunk partials of this rank's key shard from the fp64 oracle."""
    import oracle
    from seeded_inputs import bf16_bits
    orc = oracle.get()
    B, H, _, d = q.shape
    o = torch.zeros((B, H, S, d), dtype=torch.float64)
    lse = torch.zeros((B, H, S), dtype=torch.float64)
    for b in range(B):
        for h in range(H):
            ro, rl = orc.decode_partials_bf16(bf16_bits(q[b, h, 0]), bf16_bits(k[b, h]),
                                              bf16_bits(v[b, h]), scale, S)
            o[b, h], lse[b, h] = torch.from_numpy(ro), torch.from_numpy(rl)
    return o, lse


def _oracle_merge(og, lg):
    """The oracle's max-and-sum merge over all R x S gathered chunks of each row."""
    import oracle
    orc = oracle.get()
    R, B, H, S, d = og.shape
    o = np.zeros((B, H, d))
    lse = np.zeros((B, H))
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = orc.lse_merge_f64(og[:, b, h].reshape(R * S, d).numpy(),
                                                   lg[:, b, h].reshape(R * S).numpy())
    return o, lse


def _worker(rank, world, port, out, B, H, Nkv, d, S):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from seeded_inputs import bf16_bits, make_qkv
        scale = float(np.float32(1.0 / np.sqrt(d)))
        q, k, v = make_qkv(B, H, 1, Nkv, d, seed=31)      # the same full draw on every rank
        lo, hi = kv_range(Nkv, rank, world)
        o, lse = kv_split_decode(q, k[:, :, lo:hi].contiguous(), v[:, :, lo:hi].contiguous(),
                                 scale, S, _oracle_partials, _oracle_merge)
        o_full, l_full = oracle.get().attn_fwd_bf16(bf16_bits(q), bf16_bits(k), bf16_bits(v),
                                                    False, scale)
        dec_err = (float(np.abs(o - o_full[:, :, 0]).max()), float(np.abs(lse - l_full[:, :, 0]).max()))
        # prefill: heads partitioned over the ranks, each computes its range only
        qp, kp, vp = make_qkv(2, 3, 40, 40, 16, seed=32)
        a, b_ = head_range(2, 3, rank, world)
        flat = [t.reshape(6, 1, 40, 16)[a:b_].reshape(1, b_ - a, 40, 16) for t in (qp, kp, vp)]
        o_mine, _ = oracle.get().attn_fwd_bf16(*(bf16_bits(t.contiguous()) for t in flat), True, 0.25)
        pieces = [None] * world
        dist.all_gather_object(pieces, (a, b_, o_mine))
        o_pf, _ = oracle.get().attn_fwd_bf16(bf16_bits(qp), bf16_bits(kp), bf16_bits(vp), True, 0.25)
        assembled = np.concatenate([p[2].reshape(p[1] - p[0], 40, 16) for p in pieces])
        pf_err = float(np.abs(assembled - o_pf.reshape(6, 40, 16)).max())
        t = max_over_ranks([1.0 + rank, 5.0 - rank])
        out[rank] = (dec_err, pf_err, (lo, hi), t)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,Nkv,S", [(2, 1000, 4), (3, 101, 8)])
def test_kv_split_decode_on_gloo_ranks_equals_unsplit(world, Nkv, S):
    """world 3 over 101 keys with 8 chunks a rank: shards of 34/34/33 keys and
    some chunks short or empty."""
    port = 29500 + (os.getpid() + world) % 1000
    B, H, d = 2, 3, 64
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out, B, H, Nkv, d, S), nprocs=world,
                           start_method="spawn")
        res = [out[r] for r in range(world)]
    assert [r[2] for r in res] == [kv_range(Nkv, r, world) for r in range(world)]
    for dec_err, pf_err, _, t in res:
        assert dec_err[0] <= 1e-12 and dec_err[1] <= 1e-12, dec_err
        assert pf_err == 0.0
        assert t == [float(world), 5.0]                 # element-wise max over ranks


def test_query_draw_does_not_depend_on_the_key_count():
    """Every rank of the split decode draws the same query rows from the base
    seed without drawing the whole sequence's keys: the queries are the
    generator's first draw, so they do not depend on how many keys follow."""
    from seeded_inputs import make_qkv
    q_small = make_qkv(2, 3, 1, 1, 16, seed=4)[0]
    q_full = make_qkv(2, 3, 1, 4097, 16, seed=4)[0]
    assert torch.equal(q_small, q_full)


def test_paged_query_draw_does_not_depend_on_the_cache_size():
    from seeded_inputs import make_paged_cache
    q_small = make_paged_cache(2, 3, [1, 1], 16, 16, seed=5)[0]
    q_full = make_paged_cache(2, 3, [300, 77], 16, 16, seed=5)[0]
    assert torch.equal(q_small, q_full)
