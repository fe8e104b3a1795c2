"""The fp64 oracle pinned to facts that do not come from itself (CPU only)."""
import pytest

import oracle
from tests import pins


def _make(lw):
    return oracle.Oracle(lw)


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(_make)
