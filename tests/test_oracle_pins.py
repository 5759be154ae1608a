"""The CPU oracle against its pins (brute force, a library routine, closed forms, invariants)."""
import pytest

from tests.oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(oracle, pin):
    pin(oracle)
