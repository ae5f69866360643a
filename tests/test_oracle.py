"""The fp64 oracle against facts fixed by the pages and by the mathematics."""
import pytest

import oracle
from tests import oracle_pins

PINS = {p.__name__: p for p in oracle_pins.ALL_PINS}


@pytest.mark.parametrize("name", sorted(PINS))
def test_oracle_pin(name):
    PINS[name](oracle)
