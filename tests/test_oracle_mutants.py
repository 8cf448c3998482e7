"""Plant one mistake at a time in the oracle (compile-time switch, CPU only)
and check that at least one pin catches it."""
import pytest

import oracle as O
import oracle_pins as P

MUTANTS = {
    1: "scale dropped",
    2: "query and key swapped",
    3: "no diagonal forcing",
    4: "ragged last group given N keys",
    5: "base-2 log-sum-exp",
    6: "mask bits read MSB first",
    7: "no division by the normaliser",
    8: "mask ignored",
    9: "backward: -D term dropped",
    10: "backward: dk without the scale",
    11: "backward: unnormalised probabilities",
    12: "backward: dq accumulates the query",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m].replace(" ", "_"))
def test_pins_catch_planted_mistake(mutant):
    bad = O.Oracle(mutant=mutant)
    caught = []
    for check in P.ALL_CHECKS:
        try:
            check(bad)
        except (AssertionError, RuntimeError):
            caught.append(check.__name__)
    assert caught, f"no pin caught mutant {mutant} ({MUTANTS[mutant]})"
