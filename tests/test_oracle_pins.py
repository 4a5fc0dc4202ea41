"""The CPU oracle against its pins (no GPU needed)."""
import pytest

import oracle
from tests import pins


@pytest.mark.parametrize("pin", pins.PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle)
