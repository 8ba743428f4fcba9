"""The CPU oracle against hand-worked values, brute force and closed forms (no GPU)."""
import pytest

import oracle
import oracle_pins


@pytest.mark.parametrize("check", oracle_pins.ALL, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(oracle)
