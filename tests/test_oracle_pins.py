"""The fp64 oracle against facts fixed outside it (closed forms, library
routines, finite differences, decode == prefill).  CPU only."""
import pytest

import oracle
import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.load())
