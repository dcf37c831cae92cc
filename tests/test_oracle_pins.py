"""The CPU oracle against its pins (no GPU): the hand-worked example, brute
force, library reductions, closed forms and the pages' invariants."""
import pytest

import oracle as O
import oracle_pins as PINS


@pytest.mark.parametrize("pin", PINS.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(O.lib())
