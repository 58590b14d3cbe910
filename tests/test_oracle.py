"""The CPU oracle against its pins (worked examples, brute force, closed
forms, invariants, library rounding).  CPU only."""
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def ora():
    return oracle.get()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(ora, pin):
    pin(ora)
