"""The oracle against its pins (hand-worked fixtures, library routines, brute
force, closed forms, cross-agreement of the drop rule)."""
import pytest

from oracle import moe_oracle
from oracle_pins import PINS


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(moe_oracle)
