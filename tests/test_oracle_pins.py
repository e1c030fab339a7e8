"""The fp64 oracle against its pins (library routines, brute force, closed forms,
hand-worked examples).  CPU only."""
import pytest

import oracle
from tests import oracle_pins as pins


@pytest.fixture(scope="module")
def o():
    return oracle.default()


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(o, check):
    check(o)
