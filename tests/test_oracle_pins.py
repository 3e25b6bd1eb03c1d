"""The CPU oracle against what the method's definition and mathematics fix (no GPU)."""
import pytest

from tests import pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(oracle_lib, check):
    check(oracle_lib)
