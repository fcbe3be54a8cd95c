"""The fp64 oracle against its pins (CPU only)."""
import pytest

import oracle
from tests_support import pins_module

pins = pins_module()


@pytest.fixture(scope="module")
def o():
    return oracle.get()


@pytest.mark.parametrize("pin", pins.PINS, ids=lambda p: p.__name__)
def test_pin(o, pin):
    pin(o)
