"""The fp64 oracle against closed forms, worked examples, brute force and invariants."""
import pytest

import oracle
from oracle_pins import ALL_CHECKS


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("check", ALL_CHECKS, ids=[c.__name__ for c in ALL_CHECKS])
def test_pin(orc, check):
    check(orc)
