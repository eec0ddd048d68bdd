"""The oracle against its pins (CPU only)."""
import pytest

import oracle
import pins


def make(**kw):
    return oracle.Oracle(**kw)


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(make)
