"""The oracle against its pins (brute force, closed forms, invariants,
torch's bf16 rounding and the hand-worked fixtures under tests/golden/)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, oracle_default):
    pin(oracle_default)
