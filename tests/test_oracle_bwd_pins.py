"""The fp64 gradient oracle against facts outside itself (CPU only)."""
import pytest

from tests import oracle_bwd_pins as pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_gradient_oracle_pin(check):
    check(None)
