"""The CPU oracle against its pins (brute force, closed forms, invariants,
library routines, the pages' printed routing matrices)."""
import pytest

import oracle
from tests import oracle_pins


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(lib, pin):
    fails = pin(lib)
    assert not fails, "\n".join(fails)
