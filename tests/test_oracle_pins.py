"""The CPU oracle against its pins (no GPU)."""
import pytest

from oracle import saga_oracle
from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(saga_oracle)
