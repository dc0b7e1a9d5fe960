"""The CPU oracle pinned to hand-worked cases, closed forms, invariants and
exact brute force (see tests/oracle_pins.py).  CPU only."""

import pytest

from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_every_pin_collected():
    assert len(ALL_PINS) >= 15
