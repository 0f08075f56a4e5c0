"""Every planted mistake in the oracle is caught by at least one pin.

The mistakes are compiled into copies of the oracle on the CPU
(-DORACLE_MUTANT=n); the real oracle is untouched:
 1 memory term dropped          2 ties to the higher index
 3 signed instead of |x| order  4 fma operands transposed
 5 sent value left in memory    6 partner value dropped in the merge
 7 merge partner ignores round  8 output not in index order
 9 two roundings instead of one  10 hard threshold strictly above
11 residual return inverted      12 AllGather sum in reverse rank order
"""
import pytest

import oracle
import pins

MUTANTS = list(range(1, 13))


@pytest.mark.parametrize("m", MUTANTS)
def test_mutant_is_caught(m, tmp_path):
    o = oracle.mutant(m, str(tmp_path))
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"planted mistake {m} passed every pin"
