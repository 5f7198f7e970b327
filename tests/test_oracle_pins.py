"""The fp64 oracle against the pins in ``oracle_pins`` (CPU only)."""
import pytest

import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_decode_matches_forward(orc):
    P.check_decode_matches_forward(orc)
