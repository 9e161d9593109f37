"""The float64 oracle's backward pass against its pins (CPU only)."""
import pytest

import oracle
from tests import oracle_bwd_pins


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", oracle_bwd_pins.ALL_BWD_PINS, ids=lambda f: f.__name__)
def test_oracle_bwd_pin(orc, pin):
    pin(orc)
