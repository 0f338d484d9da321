"""The CPU oracle against what the pages and mathematics fix (no GPU)."""

import pytest

import oracle.mla_ref as ref
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(ref)
