"""The CPU oracle checked against independent pins (no GPU needed)."""
import pytest

import oracle.attention as O
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(pin):
    pin(O)
