"""Each planted mistake in the oracle must make at least one pin fail.

The oracle source carries a small set of deliberate errors behind
``-DORACLE_MUTANT=<n>`` (a dropped term, a wrong sign, a wrong index, a swapped
operand, ...).  Building each of them and running the pins shows that the pins
are sharp enough to catch that kind of mistake.
"""
import pytest

import oracle
from oracle_pins import ALL_PINS

MUTANTS = {
    1: "bf16 rounding keeps one mantissa bit too few",
    2: "eps added outside the square root",
    3: "sum of squares instead of the mean",
    4: "gamma dropped",
    5: "residual subtracted instead of added",
    6: "norm taken of x instead of x + residual",
    7: "every pair takes its position from row t",
    8: "frequency index off by one",
    9: "interleaved pair partner instead of rotate-half",
    10: "rotation in the wrong direction",
    11: "sign of the exponent in the sigmoid",
    12: "sigmoid without the g factor",
    13: "LayerNorm with the unbiased variance",
    14: "LayerNorm without beta",
    15: "Gumbel noise subtracted instead of added",
    16: "sampling probability without the temperature",
    17: "KV cache row and position swapped",
    18: "k written into the V cache",
    # decode-step plumbing (oracle/__init__.py, Oracle.decode_step)
    19: "decode step: SwiGLU with gate and up swapped",
    20: "decode step: rotated q reported where k belongs",
    21: "decode step: MLP-side norm with the attention-side weights",
    22: "decode step: positions one step ahead",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: f"m{m}")
def test_mutant_is_caught(mutant):
    orc = oracle.Oracle(mutant)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {mutant}: {MUTANTS[mutant]}"
