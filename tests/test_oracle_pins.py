"""The CPU oracle against facts outside itself (brute force, library routines,
closed forms, RoPE identities, bf16 rounding)."""
import pytest

import oracle.mla_oracle as O
from tests.oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(pin):
    pin(O)
