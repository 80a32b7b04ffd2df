"""GPU parity of the device bandit (draft selection; FlashSpec, Metodologia 2,
"Selecao de Rascunho via Bandit Online"; Resultados Principais, "Desempenho do
Bandit"): spec_verify_bandit_step and spec_verify_bandit_simulate, through the C
ABI, against the oracle's fp64 bandit.

The state is integer counts and sums of exact fractions, so it must match bit
for bit.  The choices are argmaxes of fp64 scores whose log, cos and sqrt come
from different libraries on the two sides (at most a few units in the last place
apart); they could differ only between two arms whose scores agree to that
precision and are not equal, which none of these seeded cases has, so the arms
are compared exactly too."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_84_b200 import binding, workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _state_of(b: "oracle.Bandit"):
    return [float(b.t[0]), float(b.arm[0]), *b.N.tolist(), *b.R.tolist()]


@pytest.mark.parametrize("policy", [binding.BANDIT_UCB1, binding.BANDIT_THOMPSON, binding.BANDIT_THOMPSON_BETA])
@pytest.mark.parametrize("K", [1, 3, 16])
def test_step_matches_oracle_every_step(policy, K):
    """400 steps of random batches (B from 0 to 3000, gamma 1-8, some steps with an
    empty batch): the device state after every step equals the oracle's."""
    rng = np.random.default_rng(1000 * policy + K)
    ref = oracle.Bandit(K, policy)
    state = binding.bandit_state(K, DEV)
    arm = torch.empty(1, dtype=torch.int32, device=DEV)
    for step in range(400):
        B = 0 if step % 37 == 5 else int(rng.integers(1, 3000))
        gamma = int(rng.integers(1, 9))
        # acceptance levels that depend on the arm, so the choice matters
        p = 0.3 + 0.5 * ((int(ref.arm[0]) + 1) % 4) / 4
        n = rng.binomial(gamma, p, size=B).astype(np.int32)
        u1 = W.draw_uniforms(rng, (K,))
        u2 = W.draw_uniforms(rng, (K,))
        want = ref.step(n, gamma, u1, u2)
        binding.bandit_step(torch.from_numpy(n).to(DEV), gamma, state, policy,
                            torch.from_numpy(u1).to(DEV), torch.from_numpy(u2).to(DEV), arm)
        got = state.cpu().tolist()
        assert got == _state_of(ref), (step, got, _state_of(ref))
        assert int(arm.item()) == want


def test_step_edge_cases():
    """No arm yet and an empty batch; NaN uniforms make every Thompson score NaN,
    so no arm wins (-1) and the next step rewards nothing; exact ties go to the
    smaller arm."""
    K = 3
    ref = oracle.Bandit(K, binding.BANDIT_THOMPSON)
    state = binding.bandit_state(K, DEV)
    seq = [([], 4), ([2, 2], 4), ([4, 0], 4), ([1, 3], 4), ([3, 3], 4), ([0, 0], 4)]
    for i, (n, g) in enumerate(seq):
        u1 = np.full(K, float("nan") if i == 4 else 0.5, np.float32)
        u2 = np.zeros(K, np.float32)
        want = ref.step(n, g, u1, u2)
        got = binding.bandit_step(torch.tensor(n, dtype=torch.int32, device=DEV), g, state,
                                  binding.BANDIT_THOMPSON, torch.from_numpy(u1).to(DEV), torch.from_numpy(u2).to(DEV))
        assert int(got.item()) == want, (i, int(got.item()), want)
        assert state.cpu().tolist() == _state_of(ref), i
        assert (want == -1) == (i == 4)
    # UCB1: three arms rewarded equally -> equal scores -> arm 0
    ref = oracle.Bandit(K, binding.BANDIT_UCB1)
    state = binding.bandit_state(K, DEV)
    for n in ([], [1], [1], [1]):
        want = ref.step(n, 1)
        got = binding.bandit_step(torch.tensor(n, dtype=torch.int32, device=DEV), 1, state, binding.BANDIT_UCB1)
        assert int(got.item()) == want
    assert want == 0 and state.cpu().tolist() == _state_of(ref)


def test_fed_by_spec_verify_on_device():
    """Three draft models (arms) of different quality over one target: each step
    verifies the chosen arm's drafts with spec_verify and feeds its n_accepted to
    the bandit on the device (only the chosen arm is read back, to pick the next
    drafts).  The oracle's bandit gets the same counts; the oracle's verification
    checks them."""
    K, B, gamma, V = 3, 8, 4, 1000
    noise = (2.5, 0.4, 1.2)  # arm 1 drafts closest to the target
    for policy in (binding.BANDIT_UCB1, binding.BANDIT_THOMPSON, binding.BANDIT_THOMPSON_BETA):
        ref = oracle.Bandit(K, policy)
        state = binding.bandit_state(K, DEV)
        rng = np.random.default_rng(5 + policy)
        arm_dev = torch.empty(1, dtype=torch.int32, device=DEV)
        u1 = W.draw_uniforms(rng, (K,))
        u2 = W.draw_uniforms(rng, (K,))
        arm = ref.step([], gamma, u1, u2)
        binding.bandit_step(torch.empty(0, dtype=torch.int32, device=DEV), gamma, state, policy,
                            torch.from_numpy(u1).to(DEV), torch.from_numpy(u2).to(DEV), arm_dev)
        assert int(arm_dev.item()) == arm
        pulls = np.zeros(K, int)
        for step in range(40):
            w = W.make_random(B, gamma, V, "bf16", seed=10_000 * policy + 100 * step + arm,
                              T=1.0, draft_noise=noise[arm])
            d = binding.to_device(w, DEV)
            _, n_dev = binding.verify(d["target"], d["draft"], d["draft_tokens"], d["temperature"],
                                      d["u_accept"], d["u_resample"])
            res = oracle.verify(w.target, w.draft, w.draft_tokens, w.temperature, w.u_accept, w.u_resample,
                                bf16=True)
            u1 = W.draw_uniforms(rng, (K,))
            u2 = W.draw_uniforms(rng, (K,))
            binding.bandit_step(n_dev, gamma, state, policy, torch.from_numpy(u1).to(DEV),
                                torch.from_numpy(u2).to(DEV), arm_dev)
            # the counts the device bandit summed, read back only to check them: equal
            # to the oracle's wherever its decision is not within rounding of a tie
            n_gpu = n_dev.cpu().numpy()
            sure = res.near_tie == 0
            assert (n_gpu[sure] == res.n_accepted[sure]).all(), step
            arm = ref.step(n_gpu, gamma, u1, u2)
            assert int(arm_dev.item()) == arm, step
            pulls[arm] += 1
        assert state.cpu().tolist() == _state_of(ref)
        assert pulls[1] == pulls.max(), pulls  # the best drafts are played most


@pytest.mark.parametrize("policy", [binding.BANDIT_UCB1, binding.BANDIT_THOMPSON, binding.BANDIT_THOMPSON_BETA])
@pytest.mark.parametrize("mu,T,runs", [((0.75, 0.6, 0.45), 10_000, 96),
                                       ((0.3, 0.5, 0.52, 0.1, 0.49), 3_001, 33),
                                       ((0.5,), 50, 5),
                                       ((0.2, 0.9), 0, 4)])
def test_simulation_matches_oracle(policy, mu, T, runs):
    """Every run's regret and final state equal the oracle's, at the pages' size
    (T = 10,000, K = 3) and at ragged ones (runs not a multiple of the 4 runs a
    CTA carries, T = 0)."""
    K = len(mu)
    U = W.bandit_uniforms(runs, T, K, seed=31 + 7 * policy + K)
    want_r, want_s = oracle.bandit_simulate(mu, T, policy, U, with_state=True)
    got_r, got_s = binding.bandit_simulate(torch.tensor(mu, dtype=torch.float64, device=DEV), T, policy,
                                           torch.from_numpy(U).to(DEV), with_state=True)
    assert got_r.cpu().numpy().tolist() == want_r.tolist()
    assert got_s.cpu().numpy().tolist() == want_s.tolist()
