"""The fp64 oracle against its independent pins (CPU only)."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_oracle_uses_threads(orc):
    assert orc.num_threads() >= 1
