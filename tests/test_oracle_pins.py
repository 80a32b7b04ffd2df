"""Pins of the CPU oracle (no GPU): closed forms, library special cases, exact
enumeration and Monte Carlo distribution tests; see ``oracle_pins.py``."""
import pytest

import oracle
import oracle_pins as P


@pytest.mark.parametrize("check", P.ALL_ORACLE_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(oracle.verify)


def test_exact_law_identities():
    P.check_exact_law_identities()


def test_distribution_ks_chi2():
    """FlashSpec, Metodologia 3 ("Equivalencia de Distribuicao"): the emitted tokens
    follow the target distribution, KS / chi-square at 0.01 over >= 10,000 trials."""
    P.check_distribution(oracle.verify)


def test_bonus_distribution():
    P.check_bonus_distribution(oracle.verify)


def test_golden_worked_example():
    """Hand-worked example (tests/golden/worked_example_v4.json)."""
    import golden_cases
    fx, a = golden_cases.worked_example_v4()
    r = oracle.verify(a["target"], a["draft"], a["draft_tokens"], a["temperature"],
                      a["u_accept"], a["u_resample"])
    for i, c in enumerate(fx["cases"]):
        assert r.n_accepted[i] == c["expect_n"], c["derivation"]
        assert list(r.out_tokens[i]) == c["expect_tokens"], c["derivation"]


try:
    from hypothesis import given, settings, strategies as st
except ImportError:  # pragma: no cover
    given = None

if given is not None:
    @settings(max_examples=60, deadline=None)
    @given(B=st.integers(1, 6), gamma=st.integers(1, 6), V=st.integers(1, 70),
           dt=st.sampled_from(["f32", "bf16"]), seed=st.integers(0, 2**30),
           temps=st.lists(st.sampled_from([0.0, 1e-3, 0.3, 1.0, 5.0]), min_size=6, max_size=6))
    def test_oracle_properties(B, gamma, V, dt, seed, temps):
        """Hypothesis edge cases (FlashSpec, Metodologia 3, "Teste Baseado em Propriedades"):
        batch sizes, speculation lengths, ragged V and temperatures incl. greedy."""
        from speculative_decoding_verification_84_b200 import workloads as W
        import oracle_pins as P
        import numpy as np
        w = W.make_random(B, gamma, V, dt, seed=seed, T=temps[:B])
        r = oracle.verify_workload(w)
        t64, d64 = w.logits_as_f64("target"), w.logits_as_f64("draft")
        for b in range(B):
            n = int(r.n_accepted[b])
            assert r.row_status[b] in (0, 8)
            assert 0 <= n <= gamma
            assert list(r.out_tokens[b, :n]) == list(w.draft_tokens[b, :n])
            assert (r.out_tokens[b, n + 1:] == -1).all()
            k = int(r.out_tokens[b, n])
            assert 0 <= k < V
            Tb = float(w.temperature[b])
            if Tb == 0.0:
                am = np.argmax(t64[b], axis=-1)
                assert k == am[n]
                assert all(w.draft_tokens[b, j] == am[j] for j in range(n))
                assert n == gamma or w.draft_tokens[b, n] != am[n]
            else:
                ln = [P.fsum_lse(t64[b, j], Tb) for j in range(gamma + 1)] + \
                     [P.fsum_lse(d64[b, j], Tb) for j in range(gamma)]
                assert np.allclose(r.log_norm[b], ln, rtol=1e-12, atol=1e-9)
