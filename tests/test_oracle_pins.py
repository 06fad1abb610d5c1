"""The CPU oracle against its pins (brute force, worked cases, closed forms,
library special cases, invariants).  No GPU needed."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin()
