"""Paged-KV split-KV decode on the B200 against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from seeded_inputs import bf16_bits, make_paged_cache
from tests import gpu_util
from tests.parity import compare

pytestmark = pytest.mark.gpu


def _run(q, kc, vc, table, lens, scale, S, num_pages=None):
    m = gpu_util.ea()
    B, H, _, d = q.shape
    o = torch.empty((B, H, 1, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, 1), dtype=torch.float32, device="cuda")
    ws = torch.empty(m.attn_decode_workspace_bytes(B, H, d, S), dtype=torch.uint8, device="cuda")
    m.attn_decode_paged(q, kc, vc, table, lens, o, lse, scale, S, ws, num_pages=num_pages)
    return o, lse, m.attn_status()


@pytest.mark.parametrize("B,H,lens,d,ps,S", [
    (3, 4, [1, 100, 4097], 128, 16, 7),
    (2, 2, [0, 300], 64, 64, 4),
    (4, 8, [5000, 2500, 17, 8192], 128, 256, 16),
    (1, 3, [1000], 64, 128, 1),
    (2, 2, [2048, 2049], 128, 1024, 64),
])
def test_paged_decode_matches_oracle(B, H, lens, d, ps, S):
    q, kc, vc, table, sl = make_paged_cache(B, H, lens, d, ps, seed=500 + sum(lens))
    scale = float(np.float32(1.0 / np.sqrt(d)))
    o, lse, st = _run(q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), sl.cuda(), scale, S)
    assert st == 0
    ro, rl = oracle.get().decode_paged_bf16(bf16_bits(q[:, :, 0]), bf16_bits(kc), bf16_bits(vc),
                                           table.numpy(), sl.numpy(), scale)
    compare(o[:, :, 0].float().cpu().numpy(), lse[:, :, 0].cpu().numpy(), ro, rl, "paged")


def test_out_of_range_pages_are_skipped_and_reported():
    """A table entry outside [0, num_pages) is never dereferenced: its keys are
    skipped and attn_status() reports ATTN_ERR_BAD_INDEX; the other rows are exact."""
    m = gpu_util.ea()
    B, H, d, ps = 2, 2, 128, 64
    q, kc, vc, table, sl = make_paged_cache(B, H, [256, 256], d, ps, seed=77)
    bad = table.clone()
    bad[1, 2] = kc.shape[0] + 1000          # sequence 1's third page is out of range
    scale = float(np.float32(1.0 / np.sqrt(d)))
    o, lse, st = _run(q.cuda(), kc.cuda(), vc.cuda(), bad.cuda(), sl.cuda(), scale, 4)
    assert st == m.ATTN_ERR_BAD_INDEX
    assert m.attn_status() == 0                          # read-and-clear
    orc = oracle.get()
    ro, rl = orc.decode_paged_bf16(bf16_bits(q[:, :, 0]), bf16_bits(kc), bf16_bits(vc),
                                   table.numpy(), sl.numpy(), scale)
    compare(o[0, :, 0].float().cpu().numpy(), lse[0, :, 0].cpu().numpy(), ro[0], rl[0], "good seq")
    # sequence 1 without its third page equals attention over the remaining three pages
    keep = np.r_[0:128, 192:256]
    kb, vb = bf16_bits(kc), bf16_bits(vc)
    for h in range(H):
        rows_k = np.stack([kb[table[1, j // ps], h, j % ps] for j in keep])
        rows_v = np.stack([vb[table[1, j // ps], h, j % ps] for j in keep])
        o1, l1 = orc.attn_rows_bf16(bf16_bits(q[1, h]), rows_k, rows_v, [0], False, scale)
        compare(o[1, h].float().cpu().numpy(), lse[1, h].cpu().numpy(), o1, l1, "skipped page")
