"""The committed CPU oracle against its pins (closed forms, reductions to
textbook attention, invariants, brute force, the page's printed figure)."""

import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS,
                         ids=[p.__name__ for p in oracle_pins.ALL_PINS])
def test_pin(orc, pin):
    pin(orc)
