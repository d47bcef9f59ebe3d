"""The fp64 oracle against closed forms, invariants and library routines (no GPU)."""
import pytest

from oracle import oracle as orc
from tests import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(orc.default())
