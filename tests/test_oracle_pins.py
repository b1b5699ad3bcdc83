"""The oracle against its pins (CPU only)."""
import pytest

import oracle
import oracle_pins as pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS + [pins.check_stored_regression],
                         ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(oracle.default())
