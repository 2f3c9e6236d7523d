"""The multi-GPU decode split's data path on one B200, ranks emulated.

Each emulated rank r holds its own dense shard of the keys (kv_range), runs
attn_decode_partials on it into slice r of one gathered buffer -- exactly what
the all-gather leaves on every GPU -- and attn_lse_merge_gathered merges the
R x S chunks. No kernel waits on another, so running the ranks' launches one
after another on one GPU is the same computation. Checked against the fp64
oracle over the whole sequence, and the merge kernel alone against the
oracle's merge of the same gathered partials.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_70_b200.sharding import kv_range
from seeded_inputs import bf16_bits, make_partials, make_qkv
from tests import gpu_util
from tests.parity import compare, compare_merge

pytestmark = pytest.mark.gpu


def _split_decode(q, k, v, scale, R, S):
    m = gpu_util.ea()
    B, H, _, d = q.shape
    og = torch.full((R, B, H, S, d), float("nan"), dtype=torch.float32, device="cuda")
    lg = torch.full((R, B, H, S), float("nan"), dtype=torch.float32, device="cuda")
    for r in range(R):
        lo, hi = kv_range(k.shape[2], r, R)
        ks, vs = k[:, :, lo:hi].contiguous(), v[:, :, lo:hi].contiguous()
        m.attn_decode_partials(q, ks, vs, og[r], lg[r], scale, S)
    o = torch.empty((B, H, 1, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, 1), dtype=torch.float32, device="cuda")
    m.attn_lse_merge_gathered(og, lg, o, lse)
    assert m.attn_status() == 0
    return o, lse, og, lg


@pytest.mark.parametrize("B,H,Nkv,d,R,S", [
    (2, 3, 5000, 128, 2, 16), (1, 4, 777, 64, 3, 8), (4, 2, 40000, 128, 8, 64),
    (2, 2, 50, 128, 8, 16),     # more chunks than keys: many empty chunks on every rank
])
def test_split_decode_matches_oracle(B, H, Nkv, d, R, S):
    q, k, v = make_qkv(B, H, 1, Nkv, d, seed=500 + Nkv)
    scale = float(np.float32(1.0 / np.sqrt(d)))
    o, lse, _, _ = _split_decode(q.cuda(), k.cuda(), v.cuda(), scale, R, S)
    o_ref, l_ref = oracle.get().attn_fwd_bf16(bf16_bits(q), bf16_bits(k), bf16_bits(v), False,
                                              scale)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, f"split decode R{R}")


@pytest.mark.parametrize("R,S,d,empty_every", [(2, 64, 128, 0), (5, 7, 64, 3), (8, 1, 128, 2)])
def test_gathered_merge_matches_oracle_merge(R, S, d, empty_every):
    m = gpu_util.ea()
    o_p, l_p = make_partials(3, 4, R * S, d, seed=600 + R, empty_every=empty_every)
    # rank r's chunks are chunks [r*S, (r+1)*S) of each row
    og = o_p.reshape(3, 4, R, S, d).permute(2, 0, 1, 3, 4).contiguous()
    lg = l_p.reshape(3, 4, R, S).permute(2, 0, 1, 3).contiguous()
    o = torch.empty((3, 4, 1, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((3, 4, 1), dtype=torch.float32, device="cuda")
    m.attn_lse_merge_gathered(og.cuda(), lg.cuda(), o, lse)
    assert m.attn_status() == 0
    ro, rl = oracle.get().lse_merge_f32in(o_p.numpy(), l_p.numpy())
    compare_merge(o[:, :, 0].float().cpu().numpy(), lse[:, :, 0].cpu().numpy(), ro, rl,
                  "gathered merge")


def test_merge_reads_unaligned_partials():
    """attn_lse_merge accepts fp32 partials that are only 4-byte aligned and bf16
    outputs that are only 2-byte aligned (the scalar-load / scalar-store path)."""
    m = gpu_util.ea()
    B, H, S, d = 2, 3, 9, 64
    o_p, l_p = make_partials(B, H, S, d, seed=610, empty_every=4)
    buf = torch.zeros(B * H * S * d + 1, dtype=torch.float32, device="cuda")
    op = buf[1:].view(B, H, S, d)
    op.copy_(o_p.cuda())
    obuf = torch.zeros(B * H * d + 1, dtype=torch.bfloat16, device="cuda")
    o = obuf[1:].view(B, H, 1, d)
    lse = torch.empty((B, H, 1), dtype=torch.float32, device="cuda")
    assert op.data_ptr() % 16 != 0 and o.data_ptr() % 8 != 0
    m.attn_lse_merge(op, l_p.cuda(), o, lse)
    assert m.attn_status() == 0
    ro, rl = oracle.get().lse_merge_f32in(o_p.numpy(), l_p.numpy())
    compare_merge(o[:, :, 0].float().cpu().numpy(), lse[:, :, 0].cpu().numpy(), ro, rl,
                  "unaligned merge")
    assert obuf[0].item() == 0.0
