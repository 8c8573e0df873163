"""The committed fp64 oracle against facts fixed by the definition
(closed forms, a library special case, brute force, finite differences,
invariants).  CPU only."""
import pytest

import oracle
from tests import oracle_pins


@pytest.fixture(scope="module")
def O():
    return oracle.default()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(O, pin):
    pin(O)
