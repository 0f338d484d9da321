"""The CPU oracle against what the pages and mathematics fix (no GPU)."""

import pytest

import oracle.mla_ref as ref
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(ref)


import oracle.append_ref as app  # noqa: E402
from append_pins import ALL_APPEND_PINS  # noqa: E402


@pytest.mark.parametrize("pin", ALL_APPEND_PINS, ids=lambda p: p.__name__)
def test_append_oracle_pin(pin):
    pin(app)


import oracle.fp8_ref as fp8  # noqa: E402
from fp8_pins import ALL_FP8_PINS  # noqa: E402


@pytest.mark.parametrize("pin", ALL_FP8_PINS, ids=lambda p: p.__name__)
def test_fp8_oracle_pin(pin):
    pin(fp8)
