"""The fp64 oracle against facts fixed by the definitions and by mathematics
(pins P1-P10, closed forms, hand-worked examples).  CPU only."""
import pytest

from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)
