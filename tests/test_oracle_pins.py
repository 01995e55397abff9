"""The fp64 oracle against closed forms, brute force, library routines, a published
test vector and hand-worked fixtures (tests/golden/).  CPU only."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__[4:])
def test_pin(pin):
    pin()
