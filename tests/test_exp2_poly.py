"""The FMA-pipe exp2 (exp2_poly_pair in ptx_sm100.cuh), emulated step by step in
fp32 on the host, stays within its stated relative error bound of 2^x.

The coefficients are read from the CUDA header, so this checks the constants
the kernel is built with. Method: round-to-nearest range reduction x = n + f
with the 1.5 * 2^23 trick, a degree-3 polynomial for 2^f on [-1/2, 1/2], and
the exponent-field add for 2^n.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_io_aware_70_b200", "csrc", "ptx_sm100.cuh")


def constants():
    text = open(HDR).read()
    c = [float(re.search(rf"kExp2C{i} = ([0-9.eE+-]+)f;", text).group(1)) for i in range(4)]
    magic = float(re.search(r"kRoundMagic = ([0-9.eE+-]+)f;", text).group(1))
    return [np.float32(x) for x in c], np.float32(magic)


def emulate(x):
    (c0, c1, c2, c3), magic = constants()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + magic).astype(np.float32)              # round to nearest even
    n = (t - magic).astype(np.float32)
    f = (n * np.float32(-1.0) + x).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-125.0, 126.0, 2_000_001, dtype=np.float64).astype(np.float32)
    y = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1e-4, rel.max()


def test_special_points():
    x = np.array([0.0, 1.0, -1.0, 8.0, -0.5, 0.5, -30.25], dtype=np.float32)
    y = emulate(x).astype(np.float64)
    assert np.all(np.abs(y / np.exp2(x.astype(np.float64)) - 1) < 1e-4)
    # masked scores (-inf) come out tiny and positive, far below any row sum
    tiny = emulate(np.array([-np.inf, -1e30, -200.0], dtype=np.float32))
    assert np.all(tiny > 0) and np.all(tiny < 1e-37)
