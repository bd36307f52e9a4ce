"""The CPU oracle against its pins (closed forms, brute force, error bounds,
hand-worked fixtures); see oracle_pins.py for what pins which function."""
import pytest

import oracle_pins
from oracle.oracle import Oracle


@pytest.fixture(scope="module")
def O():
    return Oracle()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(O, pin):
    pin(O)
