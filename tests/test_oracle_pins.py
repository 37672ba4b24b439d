"""The oracle (C and NumPy twin) against its pins: closed forms, brute force over all
levels, the CellFill invariants, packed-layout facts and the fp64 matmul vs BLAS."""
import pytest

from oracle_impls import IMPLS
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("impl", sorted(IMPLS))
@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(impl, pin):
    pin(IMPLS[impl])


def test_bruteforce_near_ties_are_rare():
    # on random data almost no quotient w/s falls within 2^-22 of a half-integer
    from oracle_pins import pin_quant_bruteforce
    assert pin_quant_bruteforce(IMPLS["c"], n_groups=40, seed=99) <= 2
