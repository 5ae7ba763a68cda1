"""The CPU oracle against closed forms, hand cases, invariants, brute force
and library routines (see ``oracle_pins``)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin()


def test_every_pin_is_collected():
    assert len(oracle_pins.ALL_PINS) >= 18
