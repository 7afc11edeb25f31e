"""The fp64 oracle against independent sources (no GPU needed)."""
import pytest

import oracle.grape_oracle as O
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(O)
