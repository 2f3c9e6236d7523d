"""The bound the backward kernel scales its fixed-point dQ accumulator by, checked
with the fp64 oracle's gradients: every partial sum of dQ_ic / scale over key
blocks, in any order, is at most 2 max|K| max_i ||dO_i|| max_j ||V_j|| (Cauchy-Schwarz with
sum_j P_ij <= 1 and O_i a convex combination of the V_j). The kernel adds a
further factor 2 for bf16 rounding; here the exact inequality must hold, and
the adversarial case shows it is tight to within a factor 2."""
import numpy as np
import pytest

import oracle


def bound(k, v, do):
    return 2 * np.abs(k).max() * np.linalg.norm(do, axis=1).max() * np.linalg.norm(v, axis=1).max()


def abs_term_sum_max(q, k, v, do, causal, scale):
    """max over (i, c) of sum_j |dS_ij K_jc|, from the oracle's P: it bounds every
    partial sum of dQ_ic / scale, whatever subset of key blocks and in whatever
    order the CTAs have added theirs."""
    o_ref, _, p = oracle.get().attn_head_f64(q, k, v, causal, scale, want_p=True)
    ds = p * (do @ v.T - np.sum(do * o_ref, axis=1, keepdims=True))
    return (np.abs(ds) @ np.abs(k)).max()


@pytest.mark.parametrize("seed,causal", [(1, False), (2, True), (3, True)])
def test_random_inputs_within_bound(seed, causal):
    rng = np.random.default_rng(seed)
    N, d = 300, 64
    q, k, v, do = (rng.standard_normal((N, d)) for _ in range(4))
    scale = 1 / np.sqrt(d)
    rq, _, _ = oracle.get().attn_bwd_head_f64(q, k, v, do, causal, scale)
    assert np.abs(rq / scale).max() <= bound(k, v, do)
    assert abs_term_sum_max(q, k, v, do, causal, scale) <= bound(k, v, do)


def test_adversarial_inputs_reach_half_the_bound():
    """Q = 0 (uniform P), V_j = (-1)^j u, dO_i = u, K_j = (-1)^j w: O = 0, D = 0,
    dS_ij = (-1)^j ||u||^2 / N and dQ_i = ||u||^2 w, half of the bound."""
    N, d = 256, 64
    rng = np.random.default_rng(5)
    u, w = rng.standard_normal(d), rng.standard_normal(d)
    sgn = (-1.0) ** np.arange(N)[:, None]
    q = np.zeros((N, d))
    v, k = sgn * u, sgn * w
    do = np.tile(u, (N, 1))
    rq, _, _ = oracle.get().attn_bwd_head_f64(q, k, v, do, False, 1.0)
    got = np.abs(rq).max()
    assert got <= bound(k, v, do)
    assert got == pytest.approx(0.5 * bound(k, v, do), rel=1e-9)
