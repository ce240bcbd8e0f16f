"""The fp64 oracle against its pins (library routines, closed forms, invariants, brute force)."""
import pytest

from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    ok, detail = pin()
    assert ok, detail
