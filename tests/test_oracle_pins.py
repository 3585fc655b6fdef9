"""The oracle against closed forms, page invariants, an independent
formulation and library routines (CPU only)."""

import pytest

from pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(pin):
    pin()
