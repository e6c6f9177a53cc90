"""The float64 oracle against its pins (CPU only). See tests/oracle_pins.py for what each pins."""
import pytest

from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()
