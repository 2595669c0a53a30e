"""The CPU oracle against its pins (no GPU)."""
import pytest

import oracle
import pins


@pytest.fixture(scope="module")
def O():
    return oracle.get()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(O, pin):
    pin(O)
