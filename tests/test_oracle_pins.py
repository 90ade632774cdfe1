"""The oracle against its pins (facts fixed by the pages and by mathematics)."""

import pytest

from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_satisfies_pin(pin):
    pin()
