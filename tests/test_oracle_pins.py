"""The CPU oracle against its pins (closed forms, library routines, brute force and
the pages' printed values). CPU only."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=[p.__name__ for p in pins.ALL_PINS])
def test_pin(pin):
    pin()
