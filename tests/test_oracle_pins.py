"""The oracle against its pins (closed forms, identities, textbook attention,
the pages' worked example).  CPU only."""
import pytest

from oracle import dart_oracle
from tests import oracle_pins


@pytest.fixture(scope="module")
def orc():
    return dart_oracle.get()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)
