"""The CPU oracle against hand-derived values, closed forms, exact integer and
exact rational arithmetic (see ``oracle_pins.py``)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(ref_oracle, pin):
    pin(ref_oracle)
