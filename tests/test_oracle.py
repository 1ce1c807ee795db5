"""The fp64 oracle against facts other than itself (closed forms, invariants,
hand-derived examples, finite differences, torch float64 SDPA + autograd)."""

import pytest

from oracle import attention as orc
from tests.oracle_pins import PINS


@pytest.mark.parametrize("name", sorted(PINS))
def test_pin(name):
    PINS[name](orc)
