"""The CPU oracle against hand-derived fixtures, library special cases, brute force and invariants."""

import pytest

import oracle_pins as P


@pytest.mark.parametrize("check", P.ALL_CHECKS, ids=lambda f: f.__name__[len("check_"):])
def test_oracle_pin(check):
    check()
