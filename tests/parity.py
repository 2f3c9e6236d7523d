"""Tolerances and comparison helpers for CUDA-vs-oracle parity.

The bar: O (bf16) within max-abs 1e-2 and mean-abs 1e-3 of the fp64 oracle;
LSE (fp32) within 1e-3 absolute. Rows with no visible key must be exactly
O = 0 and LSE = -inf on both sides.
"""
from __future__ import annotations

import numpy as np

O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """Assert parity; o_* are [..., d] arrays, lse_* [...]. Returns (max|dO|, mean|dO|, max|dLSE|)."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape, (what, o_gpu.shape, o_ref.shape)
    assert lse_gpu.shape == lse_ref.shape, (what, lse_gpu.shape, lse_ref.shape)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite O"
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), empty), f"{what}: -inf LSE rows differ"
    if empty.any():
        assert np.all(o_gpu[empty] == 0.0), f"{what}: rows with no visible key must be 0"
    d_o = np.abs(o_gpu - o_ref)
    d_l = np.abs(lse_gpu[~empty] - lse_ref[~empty])
    mx, mean = float(d_o.max(initial=0.0)), float(d_o.mean()) if d_o.size else 0.0
    ml = float(d_l.max(initial=0.0))
    assert mx <= O_MAX_ABS, f"{what}: max|dO| {mx:.3e} > {O_MAX_ABS}"
    assert mean <= O_MEAN_ABS, f"{what}: mean|dO| {mean:.3e} > {O_MEAN_ABS}"
    assert ml <= LSE_MAX_ABS, f"{what}: max|dLSE| {ml:.3e} > {LSE_MAX_ABS}"
    return mx, mean, ml
