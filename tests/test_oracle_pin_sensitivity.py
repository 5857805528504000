"""Plant a mistake in the oracle (on the CPU) and check that some pin fails.

A pin that passes whatever the oracle does pins nothing; each planted mistake
below is a plausible slip (a dropped term, a wrong index, a wrong merge) and
must be caught by at least one of the pins in oracle_pins.py.
"""
import pytest

import oracle
from tests import oracle_pins as pins

MUTATIONS = {
    oracle.MUTATION_DROP_SELF_BIT: "drop self bit",
    oracle.MUTATION_DROP_TREE: "drop tree keys",
    oracle.MUTATION_HEAD_MAP: "h % Hkv head map",
    oracle.MUTATION_NO_SCALE: "no softmax scale",
    oracle.MUTATION_BAD_MERGE: "unnormalised merge",
    oracle.MUTATION_SHORT_PREFIX: "prefix one key short",
}


@pytest.mark.parametrize("code", sorted(MUTATIONS), ids=lambda c: MUTATIONS[c])
def test_planted_mistake_is_caught(code):
    caught = []
    oracle.set_mutation(code)
    try:
        for pin in pins.ALL_PINS:
            try:
                pin()
            except (AssertionError, oracle.OracleError):
                caught.append(pin.__name__)
    finally:
        oracle.set_mutation(oracle.MUTATION_NONE)
    assert caught, f"no pin caught planted mistake {MUTATIONS[code]!r}"
