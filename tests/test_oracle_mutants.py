"""Every planted mistake in the oracle must fail at least one pin.

The oracle source has ORACLE_MUTANT switches, each planting one plausible bug
(dropped scale, wrong key index, off-by-one or mis-aligned causal mask, sign
error in the exponent, dropped normalisation, LSE without the max term,
transposed V, unnormalised merge weights, a paged decode that ignores its block
table or reads past the sequence, a backward pass without the D term or the
dK scale, an e4m3 decoder with the wrong exponent bias, an 8-bit entry that
ignores V's descale factor). Building each variant and running
the pins shows the pins would notice that mistake in the real oracle.
"""
import pytest

import oracle
from tests import oracle_pins

MUTANTS = {
    1: "dropped scale",
    2: "mirrored key index",
    3: "causal mask off by one",
    4: "causal mask top-left aligned",
    5: "sign error in the exponent",
    6: "dropped softmax normalisation",
    7: "LSE without the max term",
    8: "transposed V operand",
    9: "merge weights not normalised",
    10: "paged decode ignores the block table",
    11: "paged decode reads one token past the sequence",
    12: "backward drops the D term",
    13: "backward dK without the scale",
    14: "e4m3 exponent bias 8",
    15: "e4m3 V descale ignored",
}


@pytest.mark.parametrize("n", sorted(MUTANTS), ids=lambda n: MUTANTS[n].replace(" ", "_"))
def test_mutant_is_caught(tmp_path, n):
    bad = oracle.build_mutant(n, str(tmp_path))
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(bad)
        except (AssertionError, RuntimeError):   # a wrong answer or a refused input
            failed.append(pin.__name__)
    assert failed, f"mutant {n} ({MUTANTS[n]}) passed every pin"
