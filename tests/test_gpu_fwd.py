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
    (1, 1, 1, 5000, 128, True),     # one query row over 40 K/V tiles
    (1, 1, 2048, 2048, 128, False), # long non-causal rows: many ring wraps
    (1, 2, 1536, 4096, 64, True),   # Nq < Nkv at length
    (2, 1, 3000, 1000, 128, True),  # Nq > Nkv at length: 2000 rows per head see no key
    (8, 64, 100, 100, 128, False),  # 512 units: several persistent rounds, a partial last one
    (4, 100, 257, 257, 64, True),   # 800 units of two sizes over 5.4 rounds
    # long K/V rows: the unit order groups the heads (3 heads of 10.7 MB of K/V
    # per group, the last group short; then one head per group)
    (2, 4, 300, 21845, 128, True),
    (1, 3, 512, 65536, 128, False),
    # head dim 64 (one issuing thread per Q tile) with long K/V rows: with the
    # dynamic deal, groups of 5 heads of 5.6 MB of K/V, the last group short
    (2, 4, 300, 21845, 64, True),
]


@pytest.mark.parametrize("scale", [0.5, 0.01])
def test_fwd_other_scales(scale):
    """A larger scale sharpens the softmax (more lazy rescales); a tiny one flattens it.

    The absolute O bar (1e-2) is stated for the workloads' scale 1/sqrt(d),
    where P is spread over many keys. At scale 0.5 one key can carry most of a
    row, O then follows single values of V (|V| up to ~4.5), and the bf16
    roundings of P (relative 2^-9) and of O (2^-9) alone reach ~1.8e-2. So each
    element is held to the rounding model instead: |O - O_ref| <= 2^-8 |O_ref|
    + 8 * 2^-9 * sqrt(sum_j (P_ij V_jc)^2), with the oracle's P; LSE keeps its
    1e-3 bar."""
    import oracle
    from seeded_inputs import make_qkv
    from tests.parity import LSE_MAX_ABS
    B, H, Nq, Nkv, d = 1, 2, 700, 900, 128
    q, k, v = make_qkv(B, H, Nq, Nkv, d, 77)
    o, lse = gpu_util.run_fwd(q.cuda(), k.cuda(), v.cuda(), True, scale, guard=256)
    orc = oracle.get()
    for h in range(H):
        qh, kh, vh = (t[0, h].double().numpy() for t in (q, k, v))
        o_ref, l_ref, pm = orc.attn_head_f64(qh, kh, vh, True, scale, want_p=True)
        allowed = 2.0 ** -8 * np.abs(o_ref) + 8 * 2.0 ** -9 * np.sqrt((pm ** 2) @ (vh ** 2))
        err = np.abs(o[0, h].double().cpu().numpy() - o_ref)
        assert np.all(err <= allowed), f"scale {scale} head {h}: {int((err > allowed).sum())} elements"
        dl = np.abs(lse[0, h].double().cpu().numpy() - l_ref)
        assert dl.max() <= LSE_MAX_ABS, f"scale {scale} head {h}: max|dLSE| {dl.max():.3e}"


@pytest.mark.parametrize("shape", SWEEP, ids=lambda s: "B{}H{}q{}kv{}d{}c{}".format(*s[:5], int(s[5])))
def test_fwd_sweep(shape):
    B, H, Nq, Nkv, d, causal = shape
    gpu_util.fwd_full_parity(B, H, Nq, Nkv, d, causal, seed=100 + Nq + Nkv + d)


@pytest.fixture
def schedule(monkeypatch, request):
    """Force the forward's unit deal (the library reads EXACT_ATTN_FWD_SCHEDULE
    on every call): the dynamic queue normally serves only launches whose K/V
    exceed L2, the static deal the rest."""
    monkeypatch.setenv("EXACT_ATTN_FWD_SCHEDULE", request.param)
    return request.param


@pytest.mark.parametrize("schedule", ["dynamic", "static"], indirect=True)
@pytest.mark.parametrize("shape", [SWEEP[i] for i in (1, 6, 9, 16, 18, 19, 20, 21, 22)],
                         ids=lambda s: "B{}H{}q{}kv{}d{}c{}".format(*s[:5], int(s[5])))
def test_fwd_sweep_both_schedules(shape, schedule):
    B, H, Nq, Nkv, d, causal = shape
    gpu_util.fwd_full_parity(B, H, Nq, Nkv, d, causal, seed=100 + Nq + Nkv + d)


def test_tiny_workload():
    w = WORKLOADS["tiny"]
    gpu_util.fwd_full_parity(w.B, w.H, w.Nq, w.Nkv, w.d, w.causal, w.seed, scale=w.scale)


def test_gpt2_1k_workload_full():
    w = WORKLOADS["gpt2_1k"]
    gpu_util.fwd_full_parity(w.B, w.H, w.Nq, w.Nkv, w.d, w.causal, w.seed, scale=w.scale,
                             guard=0)


def unit_rows(N, rng):
    """Rows to check in one head of a long launch: the first and last row, one
    random row inside every 256-row work unit (so every unit of every head is
    looked at), and the two rows on either side of one random unit boundary and
    of one random 128-row tile boundary."""
    rows = {0, N - 1}
    for u in range(0, N, 256):
        rows.add(int(min(N - 1, u + rng.integers(0, 256))))
    u = int(rng.integers(1, max(2, N // 256))) * 256
    t = int(rng.integers(0, max(1, N // 256))) * 256 + 128
    rows |= {u - 1, u, t - 1, t}
    return sorted(r for r in rows if 0 <= r < N)


@pytest.mark.parametrize("name", ["prefill_8k", "prefill_16k"])
def test_long_prefill_every_head(name):
    """The full-size launch in the configuration bench.py times, checked in
    every (batch, head): a head-, unit- or round-indexing mistake anywhere in
    the persistent schedule shows up as a wrong row somewhere."""
    import oracle
    from seeded_inputs import bf16_bits
    from tests.parity import compare
    w = WORKLOADS[name]
    q, k, v = make_workload(w, device="cuda")
    o, lse = gpu_util.run_fwd(q, k, v, w.causal, w.scale)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    orc = oracle.get()
    rng = np.random.default_rng(w.seed)
    qc, kc, vc, oc, lc = (t.cpu() for t in (q, k, v, o, lse))
    for b in range(w.B):
        for h in range(w.H):
            rows = unit_rows(w.Nq, rng)
            o_ref, l_ref = orc.attn_rows_bf16(bf16_bits(qc[b, h]), bf16_bits(kc[b, h]),
                                              bf16_bits(vc[b, h]), rows, w.causal, w.scale)
            compare(oc[b, h, rows].float().numpy(), lc[b, h, rows].numpy(), o_ref, l_ref,
                    f"{name} head ({b},{h})")


def test_deterministic():
    from seeded_inputs import make_qkv
    q, k, v = (t.cuda() for t in make_qkv(2, 4, 777, 777, 128, 5))
    o1, l1 = gpu_util.run_fwd(q, k, v, True, 0.088)
    o2, l2 = gpu_util.run_fwd(q, k, v, True, 0.088)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("schedule", ["dynamic"], indirect=True)
def test_concurrent_launches_on_two_streams(schedule):
    """Launches in flight at the same time on two streams take their work units
    from different queue entries, so neither steals the other's units."""
    from seeded_inputs import make_qkv
    m = gpu_util.ea()
    shapes = [(2, 8, 1000, 1000, 128, True, 41), (4, 6, 777, 777, 64, False, 42)]
    ins, outs, streams = [], [], [torch.cuda.Stream(), torch.cuda.Stream()]
    for (B, H, Nq, Nkv, d, causal, seed) in shapes:
        q, k, v = (t.cuda() for t in make_qkv(B, H, Nq, Nkv, d, seed))
        ins.append((q, k, v))
        outs.append((torch.empty_like(q), torch.empty((B, H, Nq), dtype=torch.float32,
                                                      device="cuda")))
    torch.cuda.synchronize()
    for rep in range(3):
        for i, (B, H, Nq, Nkv, d, causal, seed) in enumerate(shapes):
            q, k, v = ins[i]
            o, lse = outs[i]
            m.attn_fwd(q, k, v, o, lse, causal, float(np.float32(1 / np.sqrt(d))),
                       stream=streams[i].cuda_stream)
        torch.cuda.synchronize()
        assert m.attn_status() == 0
        for i, (B, H, Nq, Nkv, d, causal, seed) in enumerate(shapes):
            ref_o, ref_l = gpu_util.run_fwd(*ins[i], causal, float(np.float32(1 / np.sqrt(d))))
            assert torch.equal(outs[i][0], ref_o) and torch.equal(outs[i][1], ref_l), (rep, i)
