"""The float64 oracle against hand fixtures, closed forms, library routines and invariants."""

import pytest

from oracle import attention
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(attention)
