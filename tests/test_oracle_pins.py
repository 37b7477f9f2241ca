"""The CPU oracle against its pins (hand-worked fixtures, closed forms, brute force)."""
import pytest

import oracle.q4 as oq
from _pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(pin):
    pin(oq)
