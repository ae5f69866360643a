"""The fp64 backward oracle against its pins (CPU only)."""
import pytest

from oracle import attention_bwd_fp64
from tests import oracle_bwd_pins


@pytest.mark.parametrize("pin", oracle_bwd_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_backward_oracle_pin(pin):
    pin(attention_bwd_fp64)
