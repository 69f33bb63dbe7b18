"""Mutation check of the pins: each copy of the oracle with one planted
mistake (dropped term, wrong sign, transposed operand, swapped clip bounds,
greedy instead of random pivots, a wrong sign in the inverse update, a
decode step whose new token does not see itself, bins that share a pivot
stream, a binned clip to one bin's range, a temperature applied once, a
recentring mean over one bin, clips to narrower value ranges, a swapped
Philox key) must fail at least one pin.  The mistakes
are planted in the oracle's C source at compile time, on the CPU."""
import os

import pytest

import oracle
from tests import oracle_pins

MUTANTS = {
    1: "drops the subtraction of earlier factor columns",
    2: "adds instead of subtracts in the residual-diagonal update",
    3: "transposes the factor in the back substitution",
    4: "swaps the clip bounds",
    5: "takes the largest residual instead of a random pivot",
    6: "flips the sign of the rank-one inverse update",
    7: "drops the diagonal of the causal mask in the decode step",
    8: "gives every bin of an instance the instance's pivot stream",
    9: "clips the binned output to the first bin's value range",
    10: "divides the key kernel's beta by tau instead of tau squared",
    11: "recentres on the first bin's key mean instead of the instance's",
    12: "clips to the value range of the pivots' rows instead of all n rows",
    13: "clips a decode step to the cache's value range, without the new values",
    14: "swaps the seed's two words in the Philox key",
    15: "leaves the last value row out of the value range",
}


@pytest.mark.parametrize("k", sorted(MUTANTS), ids=lambda k: f"mutant{k}")
def test_pins_catch_planted_mistake(tmp_path, k):
    path = oracle.build(out_path=os.path.join(tmp_path, f"liboracle_m{k}.so"), mutant=k)
    bad = oracle.Oracle(path)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        if pin is oracle_pins.pin_philox_matches_library:
            continue  # slow and unrelated to the planted mistakes
        try:
            pin(bad)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {k} ({MUTANTS[k]})"
