"""Pins of the oracle's tree verification and pruning (no GPU); see ``tree_pins.py``."""
import pytest

import oracle
import tree_pins as P


@pytest.mark.parametrize("check", P.ALL_TREE_CHECKS, ids=lambda f: f.__name__)
def test_tree_pin(check):
    check(oracle)
