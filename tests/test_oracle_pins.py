"""The oracle against facts outside itself (runs on CPU)."""

import pytest

import oracle_pins
from oracle import ref


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(check):
    check(ref)
