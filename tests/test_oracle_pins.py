"""The CPU oracle against its pins (worked examples, closed forms, library
routines, brute force on tiny inputs)."""
import pytest

from oracle import moe_oracle
from tests.oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(pin):
    pin(moe_oracle)
