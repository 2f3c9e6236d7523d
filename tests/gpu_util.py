"""Helpers for the GPU parity tests: run the CUDA path, run the oracle, compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from seeded_inputs import bf16_bits, make_qkv
from tests.parity import compare


def ea():
    import exact_io_aware_70_b200 as m
    return m


def run_fwd(q, k, v, causal, scale, guard=0):
    """Run attn_fwd on device tensors; optional canary guard bands around the outputs."""
    m = ea()
    B, H, Nq, d = q.shape
    if guard:
        o_buf = torch.full((2 * guard + B * H * Nq * d,), -77.0, dtype=torch.bfloat16,
                           device=q.device)
        l_buf = torch.full((2 * guard + B * H * Nq,), -77.0, dtype=torch.float32, device=q.device)
        o = o_buf[guard:guard + B * H * Nq * d].view(B, H, Nq, d)
        lse = l_buf[guard:guard + B * H * Nq].view(B, H, Nq)
    else:
        o = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q.device)
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    m.attn_fwd(q, k, v, o, lse, causal, scale)
    assert m.attn_status() == 0
    if guard:
        for buf, n in ((o_buf, B * H * Nq * d), (l_buf, B * H * Nq)):
            assert torch.all(buf[:guard] == -77.0) and torch.all(buf[guard + n:] == -77.0), \
                "write outside the output tensor"
    return o, lse


def fwd_full_parity(B, H, Nq, Nkv, d, causal, seed, scale=None, guard=256):
    scale = float(np.float32(1.0 / np.sqrt(d))) if scale is None else scale
    q, k, v = make_qkv(B, H, Nq, Nkv, d, seed)
    o, lse = run_fwd(q.cuda(), k.cuda(), v.cuda(), causal, scale, guard=guard)
    o_ref, lse_ref = oracle.get().attn_fwd_bf16(bf16_bits(q), bf16_bits(k), bf16_bits(v),
                                                causal, scale)
    return compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref,
                   f"fwd B{B} H{H} Nq{Nq} Nkv{Nkv} d{d} causal{int(causal)}")


def sample_rows(N, rng, extra=24):
    base = {0, 1, 2, 127, 128, 129, 255, 256, 257, N // 2, N - 257, N - 256, N - 129, N - 128,
            N - 2, N - 1}
    rows = sorted({r for r in base if 0 <= r < N} | set(rng.integers(0, N, size=extra).tolist()))
    return rows


def fwd_sampled_parity(q, k, v, o, lse, causal, scale, heads, rng):
    """Oracle on sampled rows of sampled heads of a large run (tensors on device)."""
    orc = oracle.get()
    B, H, Nq, d = q.shape
    stats = []
    for (b, h) in heads:
        rows = sample_rows(Nq, rng)
        qh = bf16_bits(q[b, h].cpu())
        kh = bf16_bits(k[b, h].cpu())
        vh = bf16_bits(v[b, h].cpu())
        o_ref, l_ref = orc.attn_rows_bf16(qh, kh, vh, rows, causal, scale)
        o_g = o[b, h, rows].float().cpu().numpy()
        l_g = lse[b, h, rows].cpu().numpy()
        stats.append(compare(o_g, l_g, o_ref, l_ref, f"head ({b},{h})"))
    return stats
