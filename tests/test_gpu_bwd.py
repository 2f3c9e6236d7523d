"""Backward pass (dQ, dK, dV with recomputation) on the B200 against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from seeded_inputs import WORKLOADS, make_dout, make_qkv, make_workload
from tests import gpu_util
from tests.parity import compare_grad, grad_error_bound

pytestmark = pytest.mark.gpu


def run_bwd(q, k, v, do, causal, scale, guard=256, deterministic=False):
    """Forward then backward through the C ABI; outputs surrounded by canary bands."""
    m = gpu_util.ea()
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    o, lse = gpu_util.run_fwd(q, k, v, causal, scale)
    outs = []
    bufs = []
    for n in (B * H * Nq * d, B * H * Nkv * d, B * H * Nkv * d):
        buf = torch.full((2 * guard + n,), -77.0, dtype=torch.bfloat16, device="cuda")
        bufs.append((buf, n))
        outs.append(buf[guard:guard + n])
    dq = outs[0].view(B, H, Nq, d)
    dk = outs[1].view(B, H, Nkv, d)
    dv = outs[2].view(B, H, Nkv, d)
    ws = torch.empty(m.attn_bwd_workspace_bytes(B, H, Nq, d), dtype=torch.uint8, device="cuda")
    m.attn_bwd(q, k, v, o, do, lse, dq, dk, dv, causal, scale, ws, deterministic=deterministic)
    assert m.attn_status() == 0
    for buf, n in bufs:
        assert torch.all(buf[:guard] == -77.0) and torch.all(buf[guard + n:] == -77.0), \
            "write outside a gradient tensor"
    return dq, dk, dv, o


def check_heads(q, k, v, do, o, dq, dk, dv, causal, scale, heads, tag):
    """Compare whole heads of a run with the oracle's gradients under the error model."""
    orc = oracle.get()
    f64 = lambda t, b, h: t[b, h].double().cpu().numpy()
    for (b, h) in heads:
        qh, kh, vh, doh, oh = (f64(t, b, h) for t in (q, k, v, do, o))
        rq, rk, rv = orc.attn_bwd_head_f64(qh, kh, vh, doh, causal, scale)
        o_ref, _, p = orc.attn_head_f64(qh, kh, vh, causal, scale, want_p=True)
        bq, bk, bv = grad_error_bound(qh, kh, vh, doh, oh, p, o_ref, causal, scale)
        what = f"{tag} head ({b},{h})"
        compare_grad(f64(dq, b, h), rq, bq, "dQ " + what)
        compare_grad(f64(dk, b, h), rk, bk, "dK " + what)
        compare_grad(f64(dv, b, h), rv, bv, "dV " + what)


def _parity(B, H, Nq, Nkv, d, causal, seed):
    scale = float(np.float32(1.0 / np.sqrt(d)))
    q, k, v = (t.cuda() for t in make_qkv(B, H, Nq, Nkv, d, seed))
    do = make_dout(B, H, Nq, d, seed, device="cuda")
    dq, dk, dv, o = run_bwd(q, k, v, do, causal, scale)
    heads = [(b, h) for b in range(B) for h in range(H)]
    check_heads(q, k, v, do, o, dq, dk, dv, causal, scale, heads,
                f"B{B} H{H} Nq{Nq} Nkv{Nkv} d{d} causal{int(causal)}")


@pytest.mark.parametrize("B,H,Nq,Nkv,d,causal", [
    (1, 1, 128, 128, 64, False),      # one tile each way
    (1, 1, 128, 128, 128, True),
    (1, 2, 300, 300, 128, True),      # ragged tails on both sides
    (2, 1, 200, 520, 64, True),       # Nq < Nkv: bottom-right alignment
    (1, 1, 520, 200, 128, True),      # Nq > Nkv: leading rows see no key
    (1, 2, 1000, 777, 128, False),
    (1, 1, 1, 1, 64, False),          # single element
    (1, 1, 1, 300, 128, True),        # one query row: sees every key
    (2, 3, 640, 640, 64, False),
    (1, 2, 2048, 2048, 128, False),   # long non-causal: 32 query steps per key block
    (1, 1, 1500, 4000, 64, True),     # Nq < Nkv at length
    (1, 5, 200, 200, 128, True),      # 5 heads: a launch-order group of 4 and one of 1
    (1, 3, 333, 777, 64, False),      # 3 heads (one partial group), 7 key blocks
])
def test_bwd_matches_oracle(B, H, Nq, Nkv, d, causal):
    _parity(B, H, Nq, Nkv, d, causal, seed=Nq * 7 + Nkv + d + int(causal))


def test_bwd_other_scale():
    """scale 0.5 on d = 128 (sharper softmax): the gradients through the error model."""
    B, H, N, d = 1, 2, 600, 128
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, N, d, 91))
    do = make_dout(B, H, N, d, 91, device="cuda")
    dq, dk, dv, o = run_bwd(q, k, v, do, True, 0.5)
    check_heads(q, k, v, do, o, dq, dk, dv, True, 0.5, [(0, 0), (0, 1)], "scale 0.5")


def test_bwd_gpt2_1k_full():
    w = WORKLOADS["gpt2_1k"]
    _parity(w.B, w.H, w.Nq, w.Nkv, w.d, w.causal, w.seed)


def test_bwd_prefill_8k_one_head():
    """The full 8K x 32-head launch; the oracle checks one whole head."""
    w = WORKLOADS["prefill_8k"]
    q, k, v = make_workload(w, device="cuda")
    do = make_dout(w.B, w.H, w.Nq, w.d, w.seed, device="cuda")
    dq, dk, dv, o = run_bwd(q, k, v, do, w.causal, w.scale)
    check_heads(q, k, v, do, o, dq, dk, dv, w.causal, w.scale, [(0, 17)], "prefill_8k")


def test_bwd_dk_dv_deterministic():
    """dK and dV have a fixed summation order; attn_bwd's dQ goes through fp32 atomics."""
    scale = float(np.float32(1.0 / np.sqrt(128)))
    q, k, v = (t.cuda() for t in make_qkv(1, 4, 700, 700, 128, 11))
    do = make_dout(1, 4, 700, 128, 11, device="cuda")
    a = run_bwd(q, k, v, do, True, scale)
    b = run_bwd(q, k, v, do, True, scale)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


@pytest.mark.parametrize("d,causal", [(128, True), (64, False)])
def test_bwd_deterministic_form(d, causal):
    """attn_bwd_deterministic sums dQ in fixed point with integer atomics: every
    gradient is the same bits on every run although 256 CTAs add into dQ in
    whatever order they get there, and all three meet the error model (dK and
    dV equal attn_bwd's bit for bit)."""
    scale = float(np.float32(1.0 / np.sqrt(d)))
    B, H, N = 2, 8, 2048
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, N, d, 11 + d))
    do = make_dout(B, H, N, d, 11 + d, device="cuda")
    runs = [run_bwd(q, k, v, do, causal, scale, deterministic=True) for _ in range(3)]
    for r in runs[1:]:
        for g in range(3):
            assert torch.equal(runs[0][g], r[g]), ("dQ", "dK", "dV")[g]
    dq, dk, dv, o = runs[0]
    check_heads(q, k, v, do, o, dq, dk, dv, causal, scale, [(0, 0), (1, 7)],
                f"deterministic d{d}")
    fast = run_bwd(q, k, v, do, causal, scale)
    assert torch.equal(fast[1], dk) and torch.equal(fast[2], dv)


def test_bwd_deterministic_large_and_zero_gradients():
    """The fixed-point scale follows the inputs: large gradients (V x 8, dO x 300, so
    dQ about 2400 times its usual size; Q and K as usual, so the softmax is not
    pushed to denormal probabilities) still meet the error model without
    overflow, and dO = 0 gives exact zeros."""
    B, H, N, d = 1, 2, 400, 64
    scale = float(np.float32(1.0 / np.sqrt(d)))
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, N, d, 23))
    v = (v.float() * 8).to(torch.bfloat16)
    do = (make_dout(B, H, N, d, 23, device="cuda").float() * 300).to(torch.bfloat16)
    dq, dk, dv, o = run_bwd(q, k, v, do, True, scale, deterministic=True)
    check_heads(q, k, v, do, o, dq, dk, dv, True, scale, [(0, 0), (0, 1)], "large values")
    dq0, dk0, dv0, _ = run_bwd(q, k, v, torch.zeros_like(do), True, scale, deterministic=True)
    assert not torch.any(dq0) and not torch.any(dk0) and not torch.any(dv0)


@pytest.mark.parametrize("B,H,Nq,Nkv,d,causal", [
    (1, 2, 300, 300, 128, True),      # ragged tails
    (1, 1, 520, 200, 128, True),      # leading rows see no key
    (1, 1, 1, 1, 64, False),          # single element
])
def test_bwd_deterministic_edges(B, H, Nq, Nkv, d, causal):
    scale = float(np.float32(1.0 / np.sqrt(d)))
    seed = Nq * 3 + Nkv + d
    q, k, v = (t.cuda() for t in make_qkv(B, H, Nq, Nkv, d, seed))
    do = make_dout(B, H, Nq, d, seed, device="cuda")
    dq, dk, dv, o = run_bwd(q, k, v, do, causal, scale, deterministic=True)
    check_heads(q, k, v, do, o, dq, dk, dv, causal, scale,
                [(b, h) for b in range(B) for h in range(H)], f"deterministic {Nq}x{Nkv}")


def test_bwd_rejects_small_workspace():
    m = gpu_util.ea()
    q, k, v = (t.cuda() for t in make_qkv(1, 1, 128, 128, 64, 1))
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, 128), dtype=torch.float32, device="cuda")
    ws = torch.empty(m.attn_bwd_workspace_bytes(1, 1, 128, 64) - 256, dtype=torch.uint8,
                     device="cuda")
    with pytest.raises(m.AttnError):
        m.attn_bwd(q, k, v, o, q, lse, torch.empty_like(q), torch.empty_like(k),
                   torch.empty_like(v), False, 0.125, ws)
