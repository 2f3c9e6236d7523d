"""The fp64 oracle against its pins (closed forms, invariants, library routines)."""
import pytest

import oracle
from tests import oracle_pins


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_brute_force_scalar_loop(orc):
    """An independent scalar triple loop on a tiny causal case (extra cross-check)."""
    import math
    import numpy as np
    rng = np.random.default_rng(33)
    Nq, Nkv, d, scale = 3, 5, 2, 0.8
    q, k, v = rng.normal(size=(Nq, d)), rng.normal(size=(Nkv, d)), rng.normal(size=(Nkv, d))
    o, lse = orc.attn_head_f64(q, k, v, True, scale)
    for i in range(Nq):
        vis = [j for j in range(Nkv) if j <= i + Nkv - Nq]
        w = {j: math.exp(scale * sum(q[i][c] * k[j][c] for c in range(d))) for j in vis}
        tot = sum(w.values())
        for c in range(d):
            assert abs(o[i][c] - sum(w[j] * v[j][c] for j in vis) / tot) < 1e-12
        assert abs(lse[i] - math.log(tot)) < 1e-12
