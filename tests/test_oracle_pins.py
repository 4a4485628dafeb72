"""The CPU oracle against its pins (spec tables, library routines, brute
force, hand-computed special cases).  No GPU."""
import pytest

import oracle
import pins


@pytest.fixture(scope="module")
def O():
    return oracle.load()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(O, pin):
    pin(O)
