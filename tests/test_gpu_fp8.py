"""Forward pass on e4m3 inputs (attn_fwd_fp8) on the B200 against the fp64 oracle.

Error model (derived in the design notes): the kernel's scores are exact up to
fp32 accumulation (products of e4m3 codes are exact), so the error comes from
rounding P to e4m3 for the P V product and from the bf16 output. Per element of
O, with P the oracle's probabilities and x_v the decoded V values:
    |O - O_ref| <= 2^-8 |O_ref| + KAPPA (2^-4 M + 2^-16 M_V),
    M = sqrt(sum_j (P_ij x_v,jc)^2),  M_V = sqrt(sum_{visible j} x_v,jc^2).
e4m3 rounding is relative <= 2^-4 in its normal range; the kernel keeps each
row's largest P in [2^6, 2^8], so a subnormal P (absolute error <= 2^-10) is
at most 2^-16 of the row sum. KAPPA = 8 is about 14 sigma of the uniform
rounding; the mean error must stay under the KAPPA = 1 bound's mean. LSE
depends only on fp32 sums of unrounded P: the bf16 bar (1e-3) applies.
"""
import numpy as np
import pytest
import torch

import oracle
from seeded_inputs import WORKLOADS, fp8_codes, make_qkv_fp8
from tests import gpu_util
from tests.parity import LSE_MAX_ABS

pytestmark = pytest.mark.gpu

KAPPA = 8.0


def run_fp8(q8, k8, v8, qd, kd, vd, causal, scale, guard=256):
    m = gpu_util.ea()
    B, H, Nq, d = q8.shape
    o_buf = torch.full((2 * guard + B * H * Nq * d,), -77.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((2 * guard + B * H * Nq,), -77.0, dtype=torch.float32, device="cuda")
    o = o_buf[guard:guard + B * H * Nq * d].view(B, H, Nq, d)
    lse = l_buf[guard:guard + B * H * Nq].view(B, H, Nq)
    m.attn_fwd_fp8(q8, k8, v8, qd, kd, vd, o, lse, causal, scale)
    assert m.attn_status() == 0
    for buf, n in ((o_buf, B * H * Nq * d), (l_buf, B * H * Nq)):
        assert torch.all(buf[:guard] == -77.0) and torch.all(buf[guard + n:] == -77.0), \
            "write outside the output tensor"
    return o, lse


def check_head(o_gpu, lse_gpu, q8, k8, v8, qd, kd, vd, causal, scale, what):
    """Whole-head comparison under the error model; inputs are CPU tensors of one head."""
    orc = oracle.get()
    xq = orc.e4m3_decode(fp8_codes(q8)) * float(qd)
    xk = orc.e4m3_decode(fp8_codes(k8)) * float(kd)
    xv = orc.e4m3_decode(fp8_codes(v8)) * float(vd)
    o_ref, lse_ref, p = orc.attn_head_f64(xq, xk, xv, causal, scale, want_p=True)
    Nq, Nkv = p.shape
    vis = np.ones((Nq, Nkv))
    if causal:
        vis = (np.arange(Nkv)[None, :] <= np.arange(Nq)[:, None] + (Nkv - Nq)).astype(np.float64)
    m_p = np.sqrt((p ** 2) @ (xv ** 2))
    m_v = np.sqrt(vis @ (xv ** 2))
    bound1 = 2.0 ** -8 * np.abs(o_ref) + 2.0 ** -4 * m_p + 2.0 ** -16 * m_v
    allowed = 2.0 ** -8 * np.abs(o_ref) + KAPPA * (2.0 ** -4 * m_p + 2.0 ** -16 * m_v)
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite O"
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), empty), f"{what}: -inf LSE rows differ"
    assert np.all(o_gpu[empty] == 0.0), f"{what}: rows with no visible key must be 0"
    err = np.abs(o_gpu - o_ref)
    bad = err > allowed
    if bad.any():
        i = np.unravel_index(int(np.argmax(err - allowed)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} elements outside the error model, worst "
                             f"at {i}: got {o_gpu[i]:.6g}, oracle {o_ref[i]:.6g}, "
                             f"allowed {allowed[i]:.3g}")
    assert err.mean() <= bound1.mean(), f"{what}: mean error {err.mean():.3e} > {bound1.mean():.3e}"
    dl = np.abs(lse_gpu[~empty] - lse_ref[~empty])
    assert dl.max(initial=0.0) <= LSE_MAX_ABS, f"{what}: max|dLSE| {dl.max():.3e}"
    return float((err / np.where(allowed > 0, allowed, 1.0)).max())


def _parity(B, H, Nq, Nkv, causal, seed, d=128):
    scale = float(np.float32(1.0 / np.sqrt(d)))
    q8, k8, v8, qd, kd, vd = make_qkv_fp8(B, H, Nq, Nkv, d, seed)
    o, lse = run_fp8(*(t.cuda() for t in (q8, k8, v8, qd, kd, vd)), causal, scale)
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        for h in range(H):
            check_head(o[b, h], lse[b, h], q8[b, h], k8[b, h], v8[b, h], qd[b, h], kd[b, h],
                       vd[b, h], causal, scale, f"fp8 B{B} H{H} {Nq}x{Nkv} causal{int(causal)} ({b},{h})")


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("B,H,Nq,Nkv,causal", [
    (1, 1, 128, 128, False),
    (1, 1, 128, 128, True),
    (1, 2, 300, 300, True),       # ragged tails
    (2, 1, 200, 520, True),       # Nq < Nkv: bottom-right alignment
    (1, 1, 520, 200, True),       # Nq > Nkv: leading rows see no key
    (1, 2, 1000, 777, False),
    (1, 1, 1, 1, False),
    (1, 3, 2048, 2048, True),     # many K/V tiles per row: lazy rescaling and ring wrap
    (4, 40, 300, 300, True),      # 320 units: two or three per CTA, every second one ragged
])
def test_fp8_matches_oracle(B, H, Nq, Nkv, causal, d):
    _parity(B, H, Nq, Nkv, causal, seed=Nq * 5 + Nkv + int(causal) + d, d=d)


def test_fp8_long_noncausal_d64():
    _parity(1, 1, 4096, 4096, False, 55, d=64)


def test_fp8_gpt2_1k_full():
    """The GPT-2-style workload (B=8, H=12, N=1024, d=64, causal) in e4m3, every head."""
    w = WORKLOADS["gpt2_1k"]
    _parity(w.B, w.H, w.Nq, w.Nkv, w.causal, w.seed, d=w.d)


def test_fp8_prefill_8k_one_head():
    """The full prefill_8k shape in e4m3; the oracle checks one whole head."""
    w = WORKLOADS["prefill_8k"]
    q8, k8, v8, qd, kd, vd = make_qkv_fp8(w.B, w.H, w.Nq, w.Nkv, w.d, w.seed, device="cuda")
    o, lse = run_fp8(q8, k8, v8, qd, kd, vd, w.causal, w.scale)
    h = 9
    check_head(o[0, h].float().cpu().numpy(), lse[0, h].cpu().numpy(), q8[0, h].cpu(),
               k8[0, h].cpu(), v8[0, h].cpu(), qd[0, h].cpu(), kd[0, h].cpu(), vd[0, h].cpu(),
               w.causal, w.scale, "fp8 prefill_8k head 9")


def test_fp8_rejects_head_dim_96():
    m = gpu_util.ea()
    q8, k8, v8, qd, kd, vd = (t.cuda() for t in make_qkv_fp8(1, 1, 128, 128, 96, 1))
    o = torch.empty((1, 1, 128, 96), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 1, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(m.AttnError):
        m.attn_fwd_fp8(q8, k8, v8, qd, kd, vd, o, lse, False, 0.125)
