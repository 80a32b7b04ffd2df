"""Pins of the oracle's speculation-cache functions (no GPU); see ``topf_pins.py``."""
import pytest

import oracle
import topf_pins as P


@pytest.mark.parametrize("check", P.ALL_TOPF_CHECKS, ids=lambda f: f.__name__)
def test_topf_pin(check):
    check(oracle)
