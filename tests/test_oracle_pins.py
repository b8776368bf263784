"""The CPU oracle against its pins (page examples, closed forms, library routines,
invariants).  No GPU needed."""
import pytest

from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__[4:])
def test_pin(pin):
    pin()
