"""The float64 oracle against its pins (CPU only)."""
import pytest

import oracle
from tests.oracle_pins import LSE_PINS, MAPPED_PINS, PINS, VERIFY_PINS


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(oracle.gqa_decode)


@pytest.mark.parametrize("pin", LSE_PINS, ids=[p.__name__ for p in LSE_PINS])
def test_oracle_lse_pin(pin):
    pin(oracle.gqa_decode_lse)


@pytest.mark.parametrize("pin", VERIFY_PINS, ids=[p.__name__ for p in VERIFY_PINS])
def test_oracle_verify_pin(pin):
    pin(oracle.gqa_decode_verify)


@pytest.mark.parametrize("pin", MAPPED_PINS, ids=[p.__name__ for p in MAPPED_PINS])
def test_oracle_mapped_pin(pin):
    pin(oracle.gqa_decode_mapped)
