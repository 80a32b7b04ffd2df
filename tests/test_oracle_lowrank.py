"""Pins of the oracle's low-rank draft head (no GPU); see ``lowrank_pins.py``."""
import pytest

import oracle
import lowrank_pins as P


@pytest.mark.parametrize("check", P.ALL_LOWRANK_CHECKS, ids=lambda f: f.__name__)
def test_lowrank_pin(check):
    check(oracle)
