"""The CPU oracle against its pins (closed forms, golden words, invariants, brute force)."""
import pytest

import oracle
from tests import _pins


@pytest.mark.parametrize("pin", _pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle.default())
