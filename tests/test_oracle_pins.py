"""The fp64 oracle against worked examples, closed forms, invariants and brute force."""
import pytest

import oracle
from oracle_pins import PINS


@pytest.fixture(scope="module")
def o():
    return oracle.Oracle()


@pytest.mark.parametrize("name", sorted(PINS))
def test_pin(o, name):
    PINS[name](o)
