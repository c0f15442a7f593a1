"""The oracle against closed forms, invariants, the pages' worked example and
brute force (CPU only).  The pins themselves live in ``oracle_pins.py``."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(pin):
    pin(oracle.load())
