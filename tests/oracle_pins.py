"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError if
the oracle disagrees. ``test_oracle_pins.py`` runs them on the real oracle;
``test_oracle_mutants.py`` runs them on copies of the oracle with one planted
mistake each and requires every copy to fail at least one pin.

None of these pins re-types the oracle's own formula to compare it with itself:
they compare against hand-derived values (tests/golden), closed forms, exact
invariants, the pages' streaming recurrence (a different algorithm), and
library routines (torch's scaled_dot_product_attention and logsumexp in float64).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "closed_form_cases.json")


def _f(x):
    return float("-inf") if x == "-inf" else float(x)


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    same_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):
        diff = np.where(same_inf, 0.0, np.abs(a - b))
    assert np.all(np.isfinite(diff)) and diff.max(initial=0.0) <= tol, (
        f"{what}: max |diff| {diff.max(initial=0.0)} > {tol}")


# ---------------------------------------------------------------------------
# 1. The worked example of "Describe Flash Attention at a high level"
#    (mantramindai), section "The two ideas": one query row against T = 8 keys
#    of width d = 4, drawn from numpy's default_rng(0) in the order q, K, V, and
#    processed 2 keys at a time by the online-softmax recurrence. The page says
#    the streaming result equals the full softmax; here the full softmax is the
#    oracle, and the streaming recurrence is restated independently below.
# ---------------------------------------------------------------------------
def _streaming_attention(q, K, V, block, scale):
    """Online softmax over key blocks: running max, running sum, running output.

    Restated from the recurrence the pages describe (zenaique follow-up
    question; mantramindai "The two ideas"; hassanahmed.net online softmax):
    when a block raises the running max, the old sum and output are shrunk by
    exp(old max - new max) before the block is added.
    """
    run_max = -math.inf
    run_sum = 0.0
    run_out = np.zeros(V.shape[1])
    pos = 0
    while pos < K.shape[0]:
        blk_scores = (K[pos:pos + block] @ q) * scale
        new_max = max(run_max, float(blk_scores.max()))
        shrink = math.exp(run_max - new_max) if run_max > -math.inf else 0.0
        weights = np.exp(blk_scores - new_max)
        run_sum = run_sum * shrink + float(weights.sum())
        run_out = run_out * shrink + weights @ V[pos:pos + block]
        run_max = new_max
        pos += block
    return run_out / run_sum, run_max + math.log(run_sum)


def worked_example_inputs():
    rng = np.random.default_rng(0)
    T, d = 8, 4
    q = rng.normal(size=d)
    K = rng.normal(size=(T, d))
    V = rng.normal(size=(T, d))
    return q, K, V


def pin_worked_example(orc):
    q, K, V = worked_example_inputs()
    scale = 1.0 / math.sqrt(4)
    o_stream, lse_stream = _streaming_attention(q, K, V, block=2, scale=scale)
    o, lse = orc.attn_head_f64(q[None, :], K, V, causal=False, scale=scale)
    _close(o[0], o_stream, 1e-12, "worked example O")
    _close(lse[0], lse_stream, 1e-12, "worked example LSE")
    # other block sizes, including one block (the plain softmax) and a ragged
    # last block, give the same result
    for blk in (1, 3, 8):
        o_b, lse_b = _streaming_attention(q, K, V, block=blk, scale=scale)
        _close(o[0], o_b, 1e-12, f"worked example O, block {blk}")
        _close(lse[0], lse_b, 1e-12, f"worked example LSE, block {blk}")


# ---------------------------------------------------------------------------
# 2. Hand-derived closed forms (tests/golden/closed_form_cases.json)
# ---------------------------------------------------------------------------
def pin_golden_cases(orc):
    with open(GOLDEN) as fh:
        g = json.load(fh)
    for c in g["cases"]:
        o, lse = orc.attn_head_f64(np.array(c["q"]), np.array(c["k"]), np.array(c["v"]),
                                   causal=c["causal"], scale=c["scale"])
        _close(o, np.array(c["o"]), 1e-12, c["name"] + " O")
        _close(lse, np.array([_f(x) for x in c["lse"]]), 1e-12, c["name"] + " LSE")
    for c in g["merge_cases"]:
        o, lse = orc.lse_merge_f64(np.array(c["o_part"]),
                                   np.array([_f(x) for x in c["lse_part"]]))
        _close(o, np.array(c["o"]), 1e-12, c["name"] + " O")
        _close(lse, _f(c["lse"]), 1e-12, c["name"] + " LSE")


# ---------------------------------------------------------------------------
# 3. Exact invariants of softmax attention
# ---------------------------------------------------------------------------
def _rand(shape, seed):
    return np.random.default_rng(seed).normal(size=shape)


def pin_probabilities(orc):
    """Every row of P is a probability vector; masked entries are exactly 0."""
    for causal, (Nq, Nkv) in ((False, (9, 13)), (True, (11, 11)), (True, (5, 12))):
        q, k, v = _rand((Nq, 6), 1), _rand((Nkv, 6), 2), _rand((Nkv, 6), 3)
        o, lse, p = orc.attn_head_f64(q, k, v, causal, 0.4, want_p=True)
        assert np.all(p >= 0.0)
        _close(p.sum(axis=1), np.ones(Nq), 1e-12, "row sums of P")
        if causal:
            i = np.arange(Nq)[:, None]
            j = np.arange(Nkv)[None, :]
            assert np.all(p[j > i + (Nkv - Nq)] == 0.0), "masked entries of P"
            assert np.all(p[j <= i + (Nkv - Nq)] > 0.0), "visible entries of P"


def pin_constant_values(orc):
    """If every value row is the same vector c, every output row is c."""
    c = _rand(8, 4)
    for causal in (False, True):
        q, k = _rand((10, 8), 5), _rand((10, 8), 6)
        v = np.tile(c, (10, 1))
        o, _ = orc.attn_head_f64(q, k, v, causal, 0.35)
        _close(o, np.tile(c, (10, 1)), 1e-12, "constant V")


def pin_identical_keys(orc):
    """Identical keys: uniform weights, O = mean of V, LSE = s + ln n."""
    Nkv, d, scale = 12, 8, 0.3
    k0 = _rand(d, 7)
    q, v = _rand((4, d), 8), _rand((Nkv, d), 9)
    k = np.tile(k0, (Nkv, 1))
    o, lse = orc.attn_head_f64(q, k, v, False, scale)
    _close(o, np.tile(v.mean(axis=0), (4, 1)), 1e-12, "identical keys O")
    _close(lse, scale * (q @ k0) + math.log(Nkv), 1e-12, "identical keys LSE")


def pin_zero_query(orc):
    """q = 0: all visible scores are 0, O = mean of the visible V, LSE = ln(count)."""
    Nq, Nkv, d = 6, 9, 5
    q, k, v = np.zeros((Nq, d)), _rand((Nkv, d), 10), _rand((Nkv, d), 11)
    o, lse = orc.attn_head_f64(q, k, v, False, 0.7)
    _close(o, np.tile(v.mean(axis=0), (Nq, 1)), 1e-12, "zero query O")
    _close(lse, np.full(Nq, math.log(Nkv)), 1e-12, "zero query LSE")
    o, lse = orc.attn_head_f64(q, k, v, True, 0.7)
    for i in range(Nq):
        n = i + (Nkv - Nq) + 1
        _close(o[i], v[:n].mean(axis=0), 1e-12, f"zero query causal O row {i}")
        _close(lse[i], math.log(n), 1e-12, f"zero query causal LSE row {i}")


def pin_causal_first_row(orc):
    """Causal, Nq == Nkv: row 0 sees only key 0, so O_0 = v_0 and LSE_0 = scale q_0.k_0."""
    q, k, v = _rand((7, 6), 12), _rand((7, 6), 13), _rand((7, 6), 14)
    o, lse = orc.attn_head_f64(q, k, v, True, 0.25)
    _close(o[0], v[0], 1e-12, "causal row 0 O")
    _close(lse[0], 0.25 * float(q[0] @ k[0]), 1e-12, "causal row 0 LSE")


def pin_key_permutation(orc):
    """Non-causal attention does not depend on the order of the (key, value) pairs."""
    q, k, v = _rand((5, 6), 15), _rand((11, 6), 16), _rand((11, 6), 17)
    perm = np.random.default_rng(18).permutation(11)
    o1, l1 = orc.attn_head_f64(q, k, v, False, 0.5)
    o2, l2 = orc.attn_head_f64(q, k[perm], v[perm], False, 0.5)
    _close(o1, o2, 1e-12, "permuted keys O")
    _close(l1, l2, 1e-12, "permuted keys LSE")


def pin_value_linearity(orc):
    """O is linear in V: O(a V1 + b V2) = a O(V1) + b O(V2); LSE does not depend on V."""
    q, k = _rand((6, 4), 19), _rand((9, 4), 20)
    v1, v2 = _rand((9, 4), 21), _rand((9, 4), 22)
    for causal in (False, True):
        o1, l1 = orc.attn_head_f64(q, k, v1, causal, 0.6)
        o2, l2 = orc.attn_head_f64(q, k, v2, causal, 0.6)
        o3, l3 = orc.attn_head_f64(q, k, 2.0 * v1 - 3.0 * v2, causal, 0.6)
        _close(o3, 2.0 * o1 - 3.0 * o2, 1e-12, "linearity in V")
        _close(l1, l2, 0.0, "LSE independent of V")


def pin_causal_is_truncation(orc):
    """Causal row i (any Nq, Nkv) equals non-causal attention over keys 0..i+Nkv-Nq."""
    for Nq, Nkv in ((6, 6), (4, 9), (9, 4)):
        q, k, v = _rand((Nq, 5), 23), _rand((Nkv, 5), 24), _rand((Nkv, 5), 25)
        o, lse = orc.attn_head_f64(q, k, v, True, 0.45)
        for i in range(Nq):
            n = i + (Nkv - Nq) + 1
            if n <= 0:
                _close(o[i], np.zeros(5), 0.0, "no visible key O")
                assert lse[i] == -math.inf
                continue
            n = min(n, Nkv)
            oi, li = orc.attn_head_f64(q[i:i + 1], k[:n], v[:n], False, 0.45)
            _close(o[i], oi[0], 1e-12, f"truncation O row {i}")
            _close(lse[i], li[0], 1e-12, f"truncation LSE row {i}")


# ---------------------------------------------------------------------------
# 4. Library routines: torch scaled_dot_product_attention and logsumexp (fp64)
# ---------------------------------------------------------------------------
def pin_torch_sdpa(orc):
    F = torch.nn.functional
    for causal, (Nq, Nkv, d) in ((False, (7, 13, 8)), (True, (16, 16, 8)), (False, (1, 40, 16))):
        q, k, v = _rand((Nq, d), 26), _rand((Nkv, d), 27), _rand((Nkv, d), 28)
        scale = 1.0 / math.sqrt(d)
        o, lse = orc.attn_head_f64(q, k, v, causal, scale)
        tq, tk, tv = (torch.from_numpy(x)[None, None] for x in (q, k, v))
        ref = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
        _close(o, ref[0, 0].numpy(), 1e-12, "torch sdpa O")
        scores = (tq[0, 0] @ tk[0, 0].T) * scale
        if causal:  # square, so top-left and bottom-right alignment agree
            scores = scores.masked_fill(torch.ones(Nq, Nkv, dtype=torch.bool).triu(1),
                                        float("-inf"))
        _close(lse, torch.logsumexp(scores, dim=1).numpy(), 1e-12, "torch logsumexp LSE")


# ---------------------------------------------------------------------------
# 5. Split-KV partials and their merge
# ---------------------------------------------------------------------------
def pin_merge_any_chunking(orc):
    """Merging the per-chunk partials of any chunking gives the unsplit result."""
    from seeded_inputs import bf16_bits, make_qkv
    q, k, v = make_qkv(1, 1, 1, 37, 16, seed=29)
    qb, kb, vb = bf16_bits(q[0, 0]), bf16_bits(k[0, 0]), bf16_bits(v[0, 0])
    full_o, full_l = orc.attn_rows_bf16(qb, kb, vb, [0], False, 0.25)
    for S in (1, 2, 3, 7, 37, 64):  # 64 > 37 leaves empty chunks
        o_p, l_p = orc.decode_partials_bf16(qb[0], kb, vb, 0.25, S)
        if S > 37:
            assert np.isneginf(l_p[-1]) and np.all(o_p[-1] == 0.0)
        o, lse = orc.lse_merge_f64(o_p, l_p)
        _close(o, full_o[0], 1e-12, f"merge of {S} chunks O")
        _close(lse, full_l[0], 1e-12, f"merge of {S} chunks LSE")


def pin_partials_are_chunk_attention(orc):
    """Each partial is the exact attention of the row over its own chunk of keys."""
    from seeded_inputs import bf16_bits, make_qkv
    q, k, v = make_qkv(1, 1, 1, 20, 8, seed=30)
    qb, kb, vb = bf16_bits(q[0, 0]), bf16_bits(k[0, 0]), bf16_bits(v[0, 0])
    o_p, l_p = orc.decode_partials_bf16(qb[0], kb, vb, 0.5, 3)  # chunks of 7, 7, 6
    for c, (j0, j1) in enumerate(((0, 7), (7, 14), (14, 20))):
        oc, lc = orc.attn_rows_bf16(qb, kb[j0:j1], vb[j0:j1], [0], False, 0.5)
        _close(o_p[c], oc[0], 1e-12, f"partial {c} O")
        _close(l_p[c], lc[0], 1e-12, f"partial {c} LSE")


def pin_merge_batched_matches_single(orc):
    """The batched float-input merge equals the single merge on widened inputs."""
    from seeded_inputs import make_partials
    o_p, l_p = make_partials(2, 3, 5, 4, seed=31, empty_every=3)
    o, lse = orc.lse_merge_f32in(o_p.numpy(), l_p.numpy())
    for b in range(2):
        for h in range(3):
            o1, l1 = orc.lse_merge_f64(o_p[b, h].double().numpy(), l_p[b, h].double().numpy())
            _close(o[b, h], o1, 0.0, "batched merge O")
            _close(lse[b, h], l1, 0.0, "batched merge LSE")


# ---------------------------------------------------------------------------
# 6. bf16 entry: exact widening, same result as the double entry
# ---------------------------------------------------------------------------
def pin_bf16_entry(orc):
    from seeded_inputs import bf16_bits, make_qkv
    q, k, v = make_qkv(2, 2, 9, 11, 8, seed=32)
    o, lse = orc.attn_fwd_bf16(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, 0.3)
    for b in range(2):
        for h in range(2):
            o1, l1 = orc.attn_head_f64(q[b, h].double().numpy(), k[b, h].double().numpy(),
                                       v[b, h].double().numpy(), True, 0.3)
            _close(o[b, h], o1, 0.0, "bf16 entry O")
            _close(lse[b, h], l1, 0.0, "bf16 entry LSE")
    # the row-sampled entry is the same definition at the listed rows
    rows = [0, 4, 8]
    o_r, l_r = orc.attn_rows_bf16(bf16_bits(q[1, 0]), bf16_bits(k[1, 0]), bf16_bits(v[1, 0]),
                                  rows, True, 0.3)
    _close(o_r, o[1, 0][rows], 0.0, "row entry O")
    _close(l_r, lse[1, 0][rows], 0.0, "row entry LSE")
    # widening is exact on known bit patterns: 1.0, -2.0, 0.15625
    one = np.array([[0x3F80, 0xC000, 0x3E20]], dtype=np.uint16)
    z = np.zeros((1, 3), dtype=np.uint16)
    o_w, _ = orc.attn_rows_bf16(z, z, one, [0], False, 1.0)
    _close(o_w[0], [1.0, -2.0, 0.15625], 0.0, "bf16 widening")


# ---------------------------------------------------------------------------
# 7. Paged-KV decode (the serving variant of split-KV decode)
# ---------------------------------------------------------------------------
def _paged_layout(k, v, lens, page_size, perm_seed=None):
    """Scatter contiguous K, V [B,H,L,d] (bf16 bits) into pages [P,H,page_size,d]
    with a block table; physical page order optionally shuffled."""
    B, H, L, d = k.shape
    max_pages = L // page_size
    num_pages = B * max_pages
    order = np.arange(num_pages)
    if perm_seed is not None:
        order = np.random.default_rng(perm_seed).permutation(num_pages)
    table = order.reshape(B, max_pages).astype(np.int32)
    kc = np.zeros((num_pages, H, page_size, d), dtype=np.uint16)
    vc = np.zeros_like(kc)
    for b in range(B):
        for i in range(max_pages):
            kc[table[b, i]] = k[b, :, i * page_size:(i + 1) * page_size]
            vc[table[b, i]] = v[b, :, i * page_size:(i + 1) * page_size]
    return kc, vc, table, np.asarray(lens, dtype=np.int32)


def pin_paged_matches_contiguous(orc):
    """Any page placement gives the attention of the row over its first seq_len keys."""
    from seeded_inputs import bf16_bits, make_qkv
    B, H, L, d, ps = 3, 2, 64, 8, 16
    q, k, v = make_qkv(B, H, 1, L, d, seed=34)
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    lens = [37, 64, 1]
    for perm in (None, 35):
        kc, vc, table, sl = _paged_layout(kb, vb, lens, ps, perm)
        o, lse = orc.decode_paged_bf16(qb[:, :, 0], kc, vc, table, sl, 0.3)
        for b in range(B):
            for h in range(H):
                n = lens[b]
                ro, rl = orc.attn_rows_bf16(qb[b, h], kb[b, h, :n], vb[b, h, :n], [0], False, 0.3)
                _close(o[b, h], ro[0], 1e-12, f"paged O b{b} h{h} perm{perm}")
                _close(lse[b, h], rl[0], 1e-12, f"paged LSE b{b} h{h} perm{perm}")


def pin_paged_golden(orc):
    """Hand-derived: 3 tokens in pages stored in swapped physical order, q = 0, so
    O is the mean of the 3 visible values and LSE = ln 3; the fourth slot holds a
    value that must never be read. A second sequence of length 0 gives 0, -inf."""
    one = np.float32(1.0)
    def bits(x):
        return np.array(x, dtype=np.float32).view(np.uint32).astype(np.uint64).__rshift__(16).astype(np.uint16)
    q = bits(np.zeros((2, 1, 2)))
    kc = bits(np.zeros((2, 1, 2, 2)))
    # physical page 1 = logical page 0 (tokens 0, 1); physical page 0 = logical page 1 (token 2, unused slot)
    vc = bits(np.array([[[[6.0, 3.0], [1000.0, 1000.0]]], [[[0.0, 3.0], [3.0, 0.0]]]], dtype=np.float32))
    table = np.array([[1, 0], [0, 1]], dtype=np.int32)
    lens = np.array([3, 0], dtype=np.int32)
    o, lse = orc.decode_paged_bf16(q, kc, vc, table, lens, float(one))
    _close(o[0, 0], [3.0, 2.0], 1e-12, "paged golden O")      # mean of (0,3), (3,0), (6,3)
    _close(lse[0, 0], math.log(3.0), 1e-12, "paged golden LSE")
    _close(o[1, 0], [0.0, 0.0], 0.0, "empty sequence O")
    assert lse[1, 0] == -math.inf


# ---------------------------------------------------------------------------
# 8. Backward pass (gradients of sum(dO * O))
# ---------------------------------------------------------------------------
def pin_bwd_torch_autograd(orc):
    """torch autograd through scaled_dot_product_attention in float64 (CPU)."""
    F = torch.nn.functional
    for causal, (Nq, Nkv, d) in ((False, (7, 11, 8)), (True, (12, 12, 4)), (False, (1, 30, 16))):
        q, k, v, do = (_rand(s_, 40 + i) for i, s_ in enumerate(((Nq, d), (Nkv, d), (Nkv, d),
                                                                  (Nq, d))))
        scale = 1.0 / math.sqrt(d)
        dq, dk, dv = orc.attn_bwd_head_f64(q, k, v, do, causal, scale)
        tq, tk, tv = (torch.from_numpy(x)[None, None].requires_grad_(True) for x in (q, k, v))
        out = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
        out.backward(torch.from_numpy(do)[None, None])
        _close(dq, tq.grad[0, 0].numpy(), 1e-10, "autograd dQ")
        _close(dk, tk.grad[0, 0].numpy(), 1e-10, "autograd dK")
        _close(dv, tv.grad[0, 0].numpy(), 1e-10, "autograd dV")


def pin_bwd_finite_differences(orc):
    """Central differences of L = sum(dO * O) through the forward oracle."""
    Nq, Nkv, d, scale = 5, 6, 3, 0.7
    q, k, v, do = _rand((Nq, d), 50), _rand((Nkv, d), 51), _rand((Nkv, d), 52), _rand((Nq, d), 53)
    for causal in (False, True):
        dq, dk, dv = orc.attn_bwd_head_f64(q, k, v, do, causal, scale)

        def loss(q_, k_, v_):
            o, _ = orc.attn_head_f64(q_, k_, v_, causal, scale)
            return float((o * do).sum())
        h = 1e-6
        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            for (a, b) in ((0, 0), (x.shape[0] - 1, d - 1), (2, 1)):
                xp, xm = x.copy(), x.copy()
                xp[a, b] += h
                xm[a, b] -= h
                args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
                args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
                num = (loss(*args_p) - loss(*args_m)) / (2 * h)
                _close(g[a, b], num, 1e-6, f"finite difference d{name}[{a},{b}] causal{causal}")


def pin_bwd_invariants(orc):
    """Softmax is unchanged by adding one vector to every key, so the key
    gradients sum to zero; with q = 0 the weights are uniform, so dV_j is the
    mean of dO over the rows (non-causal)."""
    Nq, Nkv, d = 6, 9, 4
    q, k, v, do = _rand((Nq, d), 54), _rand((Nkv, d), 55), _rand((Nkv, d), 56), _rand((Nq, d), 57)
    for causal in (False, True):
        _, dk, _ = orc.attn_bwd_head_f64(q, k, v, do, causal, 0.5)
        _close(dk.sum(axis=0), np.zeros(d), 1e-12, "sum of dK")
    _, _, dv = orc.attn_bwd_head_f64(np.zeros((Nq, d)), k, v, do, False, 0.5)
    _close(dv, np.tile(do.sum(axis=0) / Nkv, (Nkv, 1)), 1e-12, "uniform weights dV")


# ---------------------------------------------------------------------------
# 9. e4m3 (8-bit) inputs
# ---------------------------------------------------------------------------
def pin_e4m3_decode(orc):
    """All 256 codes against torch's float8_e4m3fn widening (a library routine),
    plus values fixed by the format's definition."""
    codes = np.arange(256, dtype=np.uint8)
    got = orc.e4m3_decode(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "e4m3 NaN codes"
    _close(got[~nan], ref[~nan], 0.0, "e4m3 decode vs torch")
    hand = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
            0x39: 1.125, 0x40: 2.0, 0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0}
    for c, val in hand.items():
        _close(got[c], val, 0.0, f"e4m3 code {c:#04x}")
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF])


def pin_fp8_entry(orc):
    """The 8-bit entry equals the double entry on the values the codes and
    descale factors stand for (decoded here by torch, not by the oracle)."""
    rng = np.random.default_rng(7)
    B, H, Nq, Nkv, d = 1, 2, 9, 13, 16
    for causal in (False, True):
        q8, k8, v8 = (rng.integers(0, 256, size=(B, H, n, d), dtype=np.uint8)
                      for n in (Nq, Nkv, Nkv))
        for t in (q8, k8, v8):        # keep the codes finite (no NaN pattern)
            t[(t & 0x7F) == 0x7F] = 0x38
        qd, kd, vd = (rng.uniform(0.01, 0.1, size=(B, H)).astype(np.float32) for _ in range(3))
        o, lse = orc.attn_fwd_fp8(q8, k8, v8, qd, kd, vd, causal, 0.25)

        def val(c, ds, h):
            return (torch.from_numpy(c[0, h].copy()).view(torch.float8_e4m3fn)
                    .to(torch.float64).numpy() * float(ds[0, h]))
        for h in range(H):
            ro, rl = orc.attn_head_f64(val(q8, qd, h), val(k8, kd, h), val(v8, vd, h), causal,
                                       0.25)
            _close(o[0, h], ro, 1e-12, f"fp8 entry O head {h}")
            _close(lse[0, h], rl, 1e-12, f"fp8 entry LSE head {h}")


ALL_PINS = [
    pin_worked_example, pin_golden_cases, pin_probabilities, pin_constant_values,
    pin_identical_keys, pin_zero_query, pin_causal_first_row, pin_key_permutation,
    pin_value_linearity, pin_causal_is_truncation, pin_torch_sdpa, pin_merge_any_chunking,
    pin_partials_are_chunk_attention, pin_merge_batched_matches_single, pin_bf16_entry,
    pin_paged_matches_contiguous, pin_paged_golden,
    pin_bwd_torch_autograd, pin_bwd_finite_differences, pin_bwd_invariants,
    pin_e4m3_decode, pin_fp8_entry,
]
