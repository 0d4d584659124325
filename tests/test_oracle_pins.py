"""The oracle against its pins (CPU only)."""
import pytest

import oracle as orc
from tests import oracle_pins as pins


@pytest.fixture(scope="module")
def lib():
    return orc._load()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, lib):
    pin(lib)
