"""The oracle against the pins of tests/pins.py (CPU only)."""
import pytest

import pins
from oracle import default


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(default())
