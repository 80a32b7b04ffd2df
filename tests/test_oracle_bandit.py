"""Pins of the oracle's draft-selection bandit (no GPU); see ``bandit_pins.py``."""
import pytest

import oracle
import bandit_pins as P


@pytest.mark.parametrize("check", P.ALL_BANDIT_CHECKS, ids=lambda f: f.__name__)
def test_bandit_pin(check):
    check(lambda K, policy: oracle.Bandit(K, policy))


@pytest.mark.parametrize("check", P.ALL_SIM_CHECKS, ids=lambda f: f.__name__)
def test_bandit_sim_pin(check):
    check(lambda mu, T, policy, U: oracle.bandit_simulate(mu, T, policy, U, with_state=True),
          lambda K, policy: oracle.Bandit(K, policy))
