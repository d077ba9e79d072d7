"""The CPU oracle against its pins (no GPU)."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.PINS, ids=[p.__name__ for p in pins.PINS])
def test_pin(oracle, pin):
    pin(oracle)
