"""The FP8 oracle against its pins (tests/oracle_fp8_pins.py)."""
import pytest

from oracle import fp8
from tests import oracle_fp8_pins as pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(check):
    check(fp8)
