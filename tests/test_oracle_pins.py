"""The oracle against its pins (CPU only): see ``oracle_pins.py``."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(oracle_impl, pin):
    pin(oracle_impl)
