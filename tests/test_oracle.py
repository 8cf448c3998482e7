"""The CPU oracle against its pins (no GPU)."""
import pytest

import oracle_pins as P


@pytest.mark.parametrize("check", P.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(oracle, check):
    check(oracle)
