"""The oracle against values fixed by the pages and by the mathematics (CPU)."""
import pytest

import oracle as O
from oracle_pins import ALL_PINS


@pytest.fixture(scope="module")
def lib():
    return O.load()


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, lib):
    pin(lib)
