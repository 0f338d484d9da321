"""The scheduler oracle against its hand-worked example and invariants (no GPU)."""

import pytest

import oracle.sched_ref as sched
from sched_pins import ALL_SCHED_PINS


@pytest.mark.parametrize("pin", ALL_SCHED_PINS, ids=lambda p: p.__name__)
def test_sched_pin(pin):
    pin(sched)
