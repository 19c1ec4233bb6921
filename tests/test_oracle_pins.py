"""The fp64 oracle against its pins (hand-worked fixtures, closed forms,
brute force, invariants and library routines); see pins.py."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()
