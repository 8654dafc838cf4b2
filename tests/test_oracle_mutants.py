"""Plant one mistake at a time in the oracle (compile-time switch, CPU only)
and check that at least one pin fails for each: the pins are strong enough to
catch a dropped term, a wrong sign, a wrong index or a swapped operand."""
import pytest

import oracle
import pins

MUTANTS = {
    1: "Abar sign flipped",
    2: "readout before the state update",
    3: "D skip dropped",
    4: "gate applied to C.h only",
    5: "softplus biased",
    6: "sigmoid in place of silu",
    7: "delta bias dropped",
    8: "input x dropped from the update",
    9: "B used as the readout vector",
    10: "h0 ignored",
    11: "B, C taken from the previous token",
    12: "elementwise A from the previous token",
    13: "backward: state gradient not carried through Abar",
    14: "backward: Delta's input-term gradient dropped",
    15: "backward: sigmoid in place of the silu derivative",
    16: "zero-order hold: the A = 0 limit Delta*B lost",
    17: "conv front-end: taps reversed",
    18: "conv front-end: bias dropped",
    19: "conv front-end: window shifted one token",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m])
def test_mutant_is_caught(mutant):
    orc = oracle.Oracle(mutant)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {mutant} ({MUTANTS[mutant]}) passed every pin"
