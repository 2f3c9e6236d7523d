"""Split-KV decode and the LSE merge on the B200 against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from seeded_inputs import WORKLOADS, bf16_bits, make_partials, make_qkv, make_workload
from tests import gpu_util
from tests.parity import LSE_MAX_ABS, compare, compare_merge

pytestmark = pytest.mark.gpu


def _decode(q, k, v, scale, S):
    m = gpu_util.ea()
    B, H, _, d = q.shape
    o = torch.empty((B, H, 1, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, 1), dtype=torch.float32, device="cuda")
    ws = torch.empty(m.attn_decode_workspace_bytes(B, H, d, S), dtype=torch.uint8, device="cuda")
    m.attn_decode_splitkv(q, k, v, o, lse, scale, S, ws)
    assert m.attn_status() == 0
    return o, lse


@pytest.mark.parametrize("B,H,Nkv,d,S", [
    (1, 1, 1, 128, 1), (2, 3, 1000, 128, 7), (1, 2, 50, 64, 64), (2, 2, 4097, 64, 3),
    (1, 1, 3000, 128, 1), (3, 1, 777, 128, 16),
])
def test_decode_partials_match_oracle_partials(B, H, Nkv, d, S):
    m = gpu_util.ea()
    q, k, v = make_qkv(B, H, 1, Nkv, d, seed=200 + Nkv)
    scale = float(np.float32(1.0 / np.sqrt(d)))
    o_p = torch.empty((B, H, S, d), dtype=torch.float32, device="cuda")
    l_p = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    m.attn_decode_partials(q.cuda(), k.cuda(), v.cuda(), o_p, l_p, scale, S)
    assert m.attn_status() == 0
    orc = oracle.get()
    for b in range(B):
        for h in range(H):
            ro, rl = orc.decode_partials_bf16(bf16_bits(q[b, h, 0]), bf16_bits(k[b, h]),
                                              bf16_bits(v[b, h]), scale, S)
            # partials are fp32: hold them to the O bar of the bf16 output and the LSE bar
            compare(o_p[b, h].cpu().numpy(), l_p[b, h].cpu().numpy(), ro, rl, f"partials {b},{h}")


@pytest.mark.parametrize("B,H,Nkv,d,S", [(2, 3, 1000, 128, 7), (1, 2, 50, 64, 64), (4, 4, 8192, 128, 64)])
def test_decode_splitkv_full(B, H, Nkv, d, S):
    q, k, v = make_qkv(B, H, 1, Nkv, d, seed=300 + Nkv)
    scale = float(np.float32(1.0 / np.sqrt(d)))
    o, lse = _decode(q.cuda(), k.cuda(), v.cuda(), scale, S)
    o_ref, l_ref = oracle.get().attn_fwd_bf16(bf16_bits(q), bf16_bits(k), bf16_bits(v), False, scale)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "decode")


def test_decode_workload_every_row():
    """decode_32k in the launch configuration bench.py times, every one of its
    B x H = 512 query rows against the oracle (one batch entry at a time, so the
    host holds 2 x 268 MB of K/V at once)."""
    w = WORKLOADS["decode_32k"]
    q, k, v = make_workload(w, device="cuda")
    o, lse = _decode(q, k, v, w.scale, w.num_splits)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    orc = oracle.get()
    for b in range(w.B):
        ro, rl = orc.attn_fwd_bf16(bf16_bits(q[b:b + 1].cpu()), bf16_bits(k[b:b + 1].cpu()),
                                   bf16_bits(v[b:b + 1].cpu()), False, w.scale)
        compare(o[b:b + 1].float().cpu().numpy(), lse[b:b + 1].cpu().numpy(), ro, rl,
                f"decode_32k batch {b}")


@pytest.mark.parametrize("d,S,empty_every", [(128, 64, 0), (64, 9, 3), (128, 5, 1)])
def test_lse_merge_matches_oracle(d, S, empty_every):
    m = gpu_util.ea()
    o_p, l_p = make_partials(3, 4, S, d, seed=400 + S, empty_every=empty_every)
    o = torch.empty((3, 4, 1, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((3, 4, 1), dtype=torch.float32, device="cuda")
    m.attn_lse_merge(o_p.cuda(), l_p.cuda(), o, lse)
    assert m.attn_status() == 0
    ro, rl = oracle.get().lse_merge_f32in(o_p.numpy(), l_p.numpy())
    compare_merge(o[:, :, 0].float().cpu().numpy(), lse[:, :, 0].cpu().numpy(), ro, rl, "merge")


def test_decode_deterministic():
    q, k, v = (t.cuda() for t in make_qkv(4, 8, 1, 5000, 128, 6))
    o1, l1 = _decode(q, k, v, 0.0884, 16)
    o2, l2 = _decode(q, k, v, 0.0884, 16)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
