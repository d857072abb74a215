"""Pin sensitivity: each variant of the oracle with one planted mistake (built
on the CPU with -DORACLE_MUTANT=m) must fail at least one pin.

Planted mistakes: 1 ties to the higher column, 2 nibble order swapped,
3 low-rank factor V read transposed, 4 signed instead of magnitude order,
5 last input column dropped from the product, 6 the two kept values of a group
stored in descending column order, 7 N:M ties to the higher column, 8 N:M mask
bits numbered from the top of each byte."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("mutant", [1, 2, 3, 4, 5, 6, 7, 8])
def test_mutant_is_caught(mutant):
    o = oracle.Oracle(mutant=mutant)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(o)
        except (AssertionError, oracle.OracleError, IndexError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {mutant} passed every pin"
