"""Pins of the oracle's draft-selection bandit (FlashSpec, Metodologia 2, "Selecao
de Rascunho via Bandit Online"; Resultados Principais, "Desempenho do Bandit"):
hand-worked steps of UCB1 and Gaussian Thompson sampling, the reward as the
batch's accepted fraction, ties, and the regret of both policies on simulated
Bernoulli arms against Auer et al.'s UCB1 bound.  Each check takes a factory
``make(K, policy)`` of bandits with ``step(n_accepted, gamma, u1, u2)``."""
from __future__ import annotations

import math

import numpy as np

UCB1, THOMPSON, THOMPSON_BETA = 0, 1, 2


def check_reward_is_accepted_fraction(make):
    b = make(2, UCB1)
    assert b.step([], 4) == 0                  # nothing chosen yet: no reward; arm 0 first
    assert b.step([0, 1, 2, 4], 4) == 1        # arm 0 earns (0+1+2+4)/(4*4) = 7/16
    assert b.N.tolist() == [1.0, 0.0] and b.R.tolist() == [7 / 16, 0.0] and b.t[0] == 1.0
    b.step([4, 4, 3, 4], 4)                    # arm 1 earns 15/16
    assert b.N.tolist() == [1.0, 1.0] and b.R.tolist() == [7 / 16, 15 / 16] and b.t[0] == 2.0


def check_ucb1_hand_steps(make):
    """K = 2, one sequence, gamma = 1: rewards are the accepted counts 0 or 1.
    step 0: no arm yet -> arm 0.  step 1: arm 0 earns 1 (N0 = 1, R0 = 1, t = 1) ->
    arm 1 is still unrewarded.  step 2: arm 1 earns 0 (t = 2): indices
    1 + sqrt(2 ln 2) = 2.177 and 0 + 1.177 -> arm 0.  step 3: arm 0 earns 1 (N0 = 2,
    t = 3): 1 + sqrt(ln 3) = 2.048 against sqrt(2 ln 3) = 1.482 -> arm 0.  step 4:
    arm 0 earns 0 (N0 = 3, R0 = 2, t = 4): 2/3 + sqrt(2 ln 4 / 3) = 1.628 against
    sqrt(2 ln 4) = 1.665 -> arm 1."""
    b = make(2, UCB1)
    got = [b.step([], 1), b.step([1], 1), b.step([0], 1), b.step([1], 1), b.step([0], 1)]
    assert got == [0, 1, 0, 0, 1], got


def check_ties_and_unrewarded_first(make):
    b = make(3, UCB1)
    assert b.step([], 1) == 0
    assert b.step([1], 1) == 1                 # arms never rewarded come first, in order
    assert b.step([1], 1) == 2
    assert b.step([1], 1) == 0                 # equal indices: the smaller arm


def check_thompson_hand_steps(make):
    """K = 2 after one reward each (arm 0: 1, arm 1: 0).  With u1 = (1/2, 1/2),
    u2 = (0, 0): z = sqrt(2 ln 2) = 1.1774 for both, theta = (1 + 1.1774/sqrt 2,
    1.1774/sqrt 2) -> arm 0.  With u1 = (1/2, 0.999), u2 = (1/2, 0): z0 = -1.1774
    (cos pi), theta0 = 1 - 0.8326 = 0.167; z1 = sqrt(-2 ln 0.001) = 3.717,
    theta1 = 3.717 / sqrt 2 = 2.628 -> arm 1."""
    b = make(2, THOMPSON)
    b.step([], 1, [0, 0], [0, 0])
    b.step([1], 1, [0, 0], [0, 0])
    b.step([0], 1, [0, 0], [0, 0])             # now N = (1, 1), R = (1, 0), t = 2
    assert b.N.tolist() == [1.0, 1.0] and b.R.tolist() == [1.0, 0.0]
    c = make(2, THOMPSON)
    for x in ([], [1], [0]):
        c.step(x, 1, [0, 0], [0, 0])
    # the same state, two different draws for the next choice (no reward in between:
    # a step with an empty batch adds nothing)
    assert c.step([], 1, [0.5, 0.5], [0.0, 0.0]) in (0, 1)


def _simulate(make, policy, mu, T, seed):
    rng = np.random.default_rng(seed)
    b = make(len(mu), policy)
    arm = b.step([], 1, rng.random(len(mu)), rng.random(len(mu)))
    regret = 0.0
    for _ in range(T):
        regret += max(mu) - mu[arm]
        reward = int(rng.random() < mu[arm])
        arm = b.step([reward], 1, rng.random(len(mu)), rng.random(len(mu)))
    return regret


def check_regret_within_ucb1_bound(make):
    """Resultados Principais: T = 10,000 rounds, K = 3 arms; the pages' arm means
    are not given, so the bound is checked on means (0.75, 0.6, 0.45): Auer et al.
    (2002), Theorem 1: E[regret] <= sum_{D>0} 8 ln T / D + (1 + pi^2/3) sum D."""
    mu, T = (0.75, 0.6, 0.45), 10_000
    gaps = [max(mu) - m for m in mu if m < max(mu)]
    bound = sum(8 * math.log(T) / d for d in gaps) + (1 + math.pi ** 2 / 3) * sum(gaps)
    ucb = np.mean([_simulate(make, UCB1, mu, T, s) for s in range(3)])
    ts = np.mean([_simulate(make, THOMPSON, mu, T, 100 + s) for s in range(3)])
    assert ucb <= bound, (ucb, bound)
    # the pages report Thompson sampling converging faster than UCB1 (18.9 vs 100.2)
    assert ts < ucb, (ts, ucb)


def check_thompson_draw(make):
    """The choice after N = (1, 1), R = (1, 0) for two sets of uniforms."""
    def prepared():
        b = make(2, THOMPSON)
        for x in ([], [1], [0]):
            b.step(x, 1, [0, 0], [0, 0])
        return b
    # one more step carries arm 1's reward of 0 before choosing, so compute the
    # expected scores for the state after it: N = (1, 2), R = (1, 0), t = 3
    b = prepared()
    a = b.step([0], 1, [0.5, 0.5], [0.0, 0.0])
    z = math.sqrt(-2 * math.log(0.5))
    assert a == (0 if 1 + z / math.sqrt(2) > 0 + z / math.sqrt(3) else 1)
    b = prepared()
    a = b.step([0], 1, [0.5, 0.999], [0.5, 0.0])
    th0 = 1 + math.sqrt(-2 * math.log(0.5)) * math.cos(math.pi) / math.sqrt(2)
    th1 = 0 + math.sqrt(-2 * math.log(1 - 0.999)) / math.sqrt(3)
    assert a == (0 if th0 > th1 else 1) and a == 1
    # z0 = 0 (cos(pi/2)), z1 = sqrt(-2 ln 0.044) = 2.4993: theta = (1, 2.4993/sqrt 3
    # = 1.443) -> arm 1; a posterior spread of 1/(N+1) instead of 1/sqrt(N+1) would
    # give theta1 = 0.833 and pick arm 0
    b = prepared()
    assert b.step([0], 1, [0.5, 0.956], [0.25, 0.0]) == 1


def check_thompson_choice_frequency(make):
    """With N = (2, 1), R = (1, 0) the posterior draws are theta_k ~ Normal(R_k/N_k,
    1/(N_k + 1)), so arm 1 is chosen with probability Phi((0 - 1/2) / sqrt(1/3 + 1/2))
    = 0.292 (0.203 with a spread of 1/(N_k + 1)); over 20,000 draws (steps with an empty batch, which add no reward)
    the frequency stays within 5 standard errors of it."""
    b = make(2, THOMPSON)
    for x in ([], [1], [0], [0]):
        b.step(x, 1, [0, 0], [0, 0])
    assert b.N.tolist() == [2.0, 1.0] and b.R.tolist() == [1.0, 0.0]
    rng = np.random.default_rng(7)
    n, hits = 20_000, 0
    for _ in range(n):
        hits += b.step([], 1, rng.random(2), rng.random(2)) == 1
    p = 0.5 * math.erfc(0.5 / math.sqrt(1.0 / 3.0 + 0.5) / math.sqrt(2.0))
    se = math.sqrt(p * (1 - p) / n)
    assert abs(hits / n - p) < 5 * se, (hits / n, p)


def check_thompson_beta_moments(make):
    """Thompson sampling with the Beta posterior's moments.  After rewards (1, 0) on
    arm 0 and 0 on arm 1: N = (2, 1), R = (1, 0), so the posteriors are Beta(2, 2)
    and Beta(1, 2): means (1/2, 1/3), variances (1/20, 1/18).  With z0 = -0.8
    (u1 = 1 - e^-0.32, u2 = 1/2) and z1 = 0 (u2 = 1/4): theta = (1/2 - 0.8 sqrt(1/20),
    1/3) = (0.3211, 0.3333) -> arm 1 (the prior's mean: with R/N arm 1 would score 0).
    Over 20,000 draws arm 1 is chosen with probability Phi((1/3 - 1/2) /
    sqrt(1/20 + 1/18)) = 0.304 (within 5 standard errors)."""
    def prepared():
        b = make(2, THOMPSON_BETA)
        for x in ([], [1], [0], [0]):
            b.step(x, 1, [0.5, 0.5], [0.0, 0.0])
        return b
    b = prepared()
    assert b.N.tolist() == [2.0, 1.0] and b.R.tolist() == [1.0, 0.0], (b.N, b.R)
    u1 = 1.0 - math.exp(-0.32)
    assert b.step([], 1, [u1, 0.5], [0.5, 0.25]) == 1
    rng = np.random.default_rng(9)
    n, hits = 20_000, 0
    for _ in range(n):
        hits += b.step([], 1, rng.random(2), rng.random(2)) == 1
    p = 0.5 * math.erfc((0.5 - 1.0 / 3.0) / math.sqrt(1.0 / 20.0 + 1.0 / 18.0) / math.sqrt(2.0))
    se = math.sqrt(p * (1 - p) / n)
    assert abs(hits / n - p) < 5 * se, (hits / n, p)


def check_thompson_beta_regret(make):
    """The Beta-moment policy on T = 10,000 rounds of K = 3 Bernoulli arms (means
    (0.8, 0.6, 0.3)): mean regret over 6 runs below the Gaussian 1/(N+1) policy's
    and below 40 (the pages report 18.9 for their Thompson sampling)."""
    mu, T = (0.8, 0.6, 0.3), 10_000
    beta = np.mean([_simulate(make, THOMPSON_BETA, mu, T, 300 + s) for s in range(6)])
    gauss = np.mean([_simulate(make, THOMPSON, mu, T, 300 + s) for s in range(6)])
    assert beta < gauss and beta < 40.0, (beta, gauss)


ALL_BANDIT_CHECKS = [check_reward_is_accepted_fraction, check_ucb1_hand_steps, check_ties_and_unrewarded_first,
                     check_thompson_hand_steps, check_thompson_draw, check_thompson_choice_frequency,
                     check_thompson_beta_moments, check_regret_within_ucb1_bound, check_thompson_beta_regret]


# ---------------------------------------------------------------------------
# The regret simulation (``oracle.bandit_simulate``).  Each check takes
# ``sim(mu, T, policy, uniforms) -> (regret[runs], state[runs][2 + 2K])`` and the
# bandit factory ``make(K, policy)`` of the same library.

def _uniforms(runs, T, K, seed):
    from speculative_decoding_verification_84_b200.workloads import bandit_uniforms
    return bandit_uniforms(runs, T, K, seed)


def check_sim_is_composed_steps(sim, make):
    """Every run equals the loop written out with single steps: step 0 chooses from
    row 0; round s adds the gap of the arm in play, rewards it with (r_s < mu) and
    steps with row s."""
    mu, T = (0.5, 0.7, 0.62), 300
    K = len(mu)
    for policy in (UCB1, THOMPSON):
        U = _uniforms(3, T, K, 11 + policy)
        regret, state = sim(mu, T, policy, U)
        for r in range(U.shape[0]):
            b = make(K, policy)
            arm = b.step([], 1, U[r, 0, :K], U[r, 0, K:2 * K])
            reg = 0.0
            for s_ in range(1, T + 1):
                reg += max(mu) - mu[arm]
                rew = int(float(U[r, s_, 2 * K]) < mu[arm])
                arm = b.step([rew], 1, U[r, s_, :K], U[r, s_, K:2 * K])
            assert reg == regret[r], (policy, r, reg, regret[r])
            want = [b.t[0], float(arm), *b.N.tolist(), *b.R.tolist()]
            assert state[r].tolist() == want, (policy, r)


def check_sim_degenerate(sim, make):
    """One arm, or arms of equal means: no regret; every round is rewarded once."""
    T = 200
    regret, state = sim((0.4,), T, UCB1, _uniforms(2, T, 1, 3))
    assert regret.tolist() == [0.0, 0.0] and state[:, 0].tolist() == [T, T] and state[:, 2].tolist() == [T, T]
    for policy in (UCB1, THOMPSON):
        regret, state = sim((0.5, 0.5), T, policy, _uniforms(2, T, 2, 4))
        assert regret.tolist() == [0.0, 0.0] and (state[:, 2] + state[:, 3]).tolist() == [T, T]


def check_sim_regret_bound(sim, make):
    """Resultados Principais: T = 10,000, K = 3 (means (0.75, 0.6, 0.45), the pages'
    are not given): mean UCB1 regret under Auer et al.'s bound, Thompson sampling
    below UCB1, and every run's regret the sum of gap_k * N_k (N_k counts the
    rounds arm k was played, each rewarded once)."""
    mu, T, K = (0.75, 0.6, 0.45), 10_000, 3
    gaps = [max(mu) - m for m in mu]
    bound = sum(8 * math.log(T) / d for d in gaps if d > 0) + (1 + math.pi ** 2 / 3) * sum(gaps)
    ru, su = sim(mu, T, UCB1, _uniforms(8, T, K, 21))
    rt, st = sim(mu, T, THOMPSON, _uniforms(8, T, K, 22))
    assert ru.mean() <= bound, (ru.mean(), bound)
    assert rt.mean() < ru.mean(), (rt.mean(), ru.mean())
    for regret, state in ((ru, su), (rt, st)):
        for r in range(regret.size):
            N = state[r, 2:2 + K]
            assert N.sum() == T and state[r, 0] == T
            assert abs(regret[r] - sum(g * n for g, n in zip(gaps, N))) < 1e-9 * T


ALL_SIM_CHECKS = [check_sim_is_composed_steps, check_sim_degenerate, check_sim_regret_bound]
