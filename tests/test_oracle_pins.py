"""The fp64 oracle against its pins (page numbers, brute force, library, closed forms, invariants)."""

import pytest

import oracle_pins


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(oracle_lib, check):
    check(oracle_lib)
