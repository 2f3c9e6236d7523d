"""Seeded synthetic inputs shared by the oracle tests, the CUDA parity tests and bench.py.

This module holds no attention arithmetic: it only draws numbers and names the
workload shapes. Q, K and V are i.i.d. N(0, 1) rounded to bfloat16
(round-to-nearest-even, done by ``Tensor.to(torch.bfloat16)``), drawn in the
order Q, then K, then V, each as one call of ``torch.randn`` of its full
shape [B, H, N, d], from one ``torch.Generator`` seeded with ``seed``.

Two generators are available and give different (equally valid) streams:
``device="cpu"`` (used for every case the oracle checks in full) and
``device="cuda"`` (used for the multi-gigabyte workloads, where drawing on the
host would take minutes; the oracle then reads the same tensors, copied back to
the host, for the rows and heads it samples).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    """One attention workload: shapes, mask, scale and seed."""

    name: str
    B: int
    H: int
    Nq: int
    Nkv: int
    d: int
    causal: bool
    seed: int
    num_splits: int = 0  # > 0 marks a split-KV decode workload

    @property
    def scale(self) -> float:
        # the softmax temperature 1/sqrt(d), rounded to fp32 once so that the
        # GPU and the oracle (which widens this same fp32 value) agree exactly
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32))

    @property
    def is_decode(self) -> bool:
        return self.num_splits > 0


# The five synthetic workloads. Shapes follow the pages: a tiny case, the
# GPT-2-small attention shape at 1K tokens, the 8192-token 32-head case whose
# score matrix would be 134 MB per head, the 16K-context fine-tuning shape, and
# a long-context decode step over a 32K-entry KV cache split into 64 chunks.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 128, 128, 64, False, 0),
    "gpt2_1k": Workload("gpt2_1k", 8, 12, 1024, 1024, 64, True, 1),
    "prefill_8k": Workload("prefill_8k", 1, 32, 8192, 8192, 128, True, 2),
    "prefill_16k": Workload("prefill_16k", 2, 32, 16384, 16384, 128, True, 3),
    "decode_32k": Workload("decode_32k", 16, 32, 1, 32768, 128, False, 4, num_splits=64),
}

# The paged variant of decode_32k: the same 16 x 32 rows over 32768 cached tokens,
# stored in 256-token pages placed in a random physical order.
PAGED_DECODE = dict(name="decode_32k_paged", B=16, H=32, seq_len=32768, d=128, page_size=256,
                    num_splits=64, seed=5)


def make_qkv(B: int, H: int, Nq: int, Nkv: int, d: int, seed: int,
             device: str = "cpu"):
    """Draw bf16 Q [B,H,Nq,d], K [B,H,Nkv,d], V [B,H,Nkv,d] from ``seed``."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    q = torch.randn((B, H, Nq, d), generator=g, device=device, dtype=torch.float32)
    k = torch.randn((B, H, Nkv, d), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((B, H, Nkv, d), generator=g, device=device, dtype=torch.float32)
    return (q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16))


def make_dout(B: int, H: int, Nq: int, d: int, seed: int, device: str = "cpu"):
    """Draw a bf16 output gradient dO [B,H,Nq,d], i.i.d. N(0,1), from its own
    stream (``seed`` offset so that it is not a copy of Q)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed + 7919)
    return torch.randn((B, H, Nq, d), generator=g, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


def make_qkv_fp8(B: int, H: int, Nq: int, Nkv: int, d: int, seed: int, device: str = "cpu"):
    """e4m3 versions of make_qkv's draws: per (b, h) and tensor, descale =
    max|x| / 448 (rounded to fp32) and code = e4m3(x / descale) (torch's
    round-to-nearest cast, clamped to the format's +-448). Returns the codes
    [B,H,N,d] as torch.float8_e4m3fn and the descales [B,H] fp32."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = []
    for n in (Nq, Nkv, Nkv):
        x = torch.randn((B, H, n, d), generator=g, device=device, dtype=torch.float32)
        ds = (x.abs().amax(dim=(2, 3)) / 448.0).clamp_min(1e-30)
        codes = (x / ds[:, :, None, None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
        out += [codes, ds.contiguous()]
    q8, qd, k8, kd, v8, vd = out
    return q8, k8, v8, qd, kd, vd


def fp8_codes(t: torch.Tensor):
    """The raw uint8 codes of a contiguous float8_e4m3fn CPU tensor, as numpy."""
    assert t.dtype == torch.float8_e4m3fn
    return t.contiguous().view(torch.uint8).numpy()


def make_workload(w: Workload, device: str = "cpu"):
    return make_qkv(w.B, w.H, w.Nq, w.Nkv, w.d, w.seed, device=device)


def make_partials(B: int, H: int, S: int, d: int, seed: int, empty_every: int = 0):
    """Random split-KV partials (fp32 O_c [B,H,S,d], fp32 lse_c [B,H,S]).

    lse_c is N(0, 3^2) so the chunk weights span several orders of magnitude;
    with ``empty_every`` > 0 every such chunk is marked empty (lse = -inf,
    O_c = 0), the form an empty chunk takes.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    o = torch.randn((B, H, S, d), generator=g, dtype=torch.float32)
    lse = 3.0 * torch.randn((B, H, S), generator=g, dtype=torch.float32)
    if empty_every > 0:
        lse[..., ::empty_every] = float("-inf")
        o[..., ::empty_every, :] = 0.0
    return o, lse


def make_paged_cache(B: int, H: int, seq_lens, d: int, page_size: int, seed: int,
                     device: str = "cpu", spare_pages: int = 3):
    """A paged KV cache for decode: q [B,H,1,d] and K, V caches
    [num_pages, H, page_size, d], all bf16 i.i.d. N(0,1) (drawn q, K, V), with a
    block table [B, max_pages] int32 that assigns each sequence's logical pages
    to physical pages in a seeded random order, and seq_lens [B] int32.
    Unused table entries point at spare pages; spare pages hold data too."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    lens = [int(x) for x in seq_lens]
    max_pages = max(1, max((n + page_size - 1) // page_size for n in lens))
    num_pages = B * max_pages + spare_pages
    perm = torch.randperm(num_pages, generator=g)
    table = perm[:B * max_pages].reshape(B, max_pages).to(torch.int32)
    gd = torch.Generator(device=device)
    gd.manual_seed(seed)
    q = torch.randn((B, H, 1, d), generator=gd, device=device).to(torch.bfloat16)
    k = torch.randn((num_pages, H, page_size, d), generator=gd, device=device).to(torch.bfloat16)
    v = torch.randn((num_pages, H, page_size, d), generator=gd, device=device).to(torch.bfloat16)
    return q, k, v, table.to(device), torch.tensor(lens, dtype=torch.int32, device=device)


def bf16_bits(t: torch.Tensor):
    """The raw uint16 bit patterns of a contiguous bf16 CPU tensor, as numpy."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view("uint16")
