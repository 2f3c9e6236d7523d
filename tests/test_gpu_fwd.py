"""Prefill forward on the B200 against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

from seeded_inputs import WORKLOADS, make_workload
from tests import gpu_util

pytestmark = pytest.mark.gpu

SWEEP = [
    # B, H, Nq, Nkv, d, causal
    (1, 2, 1, 1, 64, False),
    (1, 1, 17, 17, 128, True),
    (2, 1, 127, 127, 64, True),
    (1, 1, 128, 128, 128, True),
    (1, 2, 129, 129, 128, False),
    (1, 1, 300, 300, 64, True),
    (1, 1, 300, 300, 128, True),
    (2, 3, 257, 513, 128, False),
    (1, 1, 100, 300, 128, True),    # fewer queries than keys: bottom-right mask
    (1, 1, 300, 100, 64, True),     # more queries than keys: rows with no visible key
    (1, 2, 1000, 1000, 128, True),
    (1, 1, 513, 513, 64, True),
    (1, 1, 64, 1000, 64, False),
    (3, 2, 384, 384, 128, False),
]


@pytest.mark.parametrize("shape", SWEEP, ids=lambda s: "B{}H{}q{}kv{}d{}c{}".format(*s[:5], int(s[5])))
def test_fwd_sweep(shape):
    B, H, Nq, Nkv, d, causal = shape
    gpu_util.fwd_full_parity(B, H, Nq, Nkv, d, causal, seed=100 + Nq + Nkv + d)


def test_tiny_workload():
    w = WORKLOADS["tiny"]
    gpu_util.fwd_full_parity(w.B, w.H, w.Nq, w.Nkv, w.d, w.causal, w.seed, scale=w.scale)


def test_gpt2_1k_workload_full():
    w = WORKLOADS["gpt2_1k"]
    gpu_util.fwd_full_parity(w.B, w.H, w.Nq, w.Nkv, w.d, w.causal, w.seed, scale=w.scale,
                             guard=0)


@pytest.mark.parametrize("name", ["prefill_8k", "prefill_16k"])
def test_long_prefill_sampled(name):
    w = WORKLOADS[name]
    q, k, v = make_workload(w, device="cuda")
    o, lse = gpu_util.run_fwd(q, k, v, w.causal, w.scale)
    rng = np.random.default_rng(w.seed)
    heads = [(0, 0), (w.B - 1, w.H - 1), (w.B // 2, w.H // 2)]
    gpu_util.fwd_sampled_parity(q, k, v, o, lse, w.causal, w.scale, heads, rng)
    # properties at every row: finite O, LSE at least the log of the visible count's lower bound
    assert torch.isfinite(o.float()).all()
    assert torch.isfinite(lse).all()


def test_deterministic():
    from seeded_inputs import make_qkv
    q, k, v = (t.cuda() for t in make_qkv(2, 4, 777, 777, 128, 5))
    o1, l1 = gpu_util.run_fwd(q, k, v, True, 0.088)
    o2, l2 = gpu_util.run_fwd(q, k, v, True, 0.088)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
