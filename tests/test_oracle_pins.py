"""The oracle against facts the mathematics fixes (see oracle_pin_battery)."""
import pytest

from oracle_pin_battery import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(orc, pin):
    pin(orc)
