"""The CPU oracle against its pins (hand-computed fixture, numpy special cases, brute force,
exact invariants, planted needles).  See tests/oracle_pins.py for what each check pins."""
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(orc, check):
    check(orc)
