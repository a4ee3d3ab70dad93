"""The CPU oracle against its pins (hand decodes, library conversions, closed forms,
brute force, invariants, the dense special case).  See ``pins.py``."""
import pytest

import oracle
import pins


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", pins.PINS, ids=lambda p: p.__name__)
def test_pin(orc, pin):
    pin(orc)
