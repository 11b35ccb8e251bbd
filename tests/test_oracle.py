"""The fp64 oracle against closed forms, invariants, brute force and torch CPU SDPA."""
import pytest

import pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check()
