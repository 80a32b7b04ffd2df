"""Each planted mistake in a copy of the oracle must fail at least one pin.

The copies are made by text substitution of ``oracle/sv_oracle.c`` into a
temporary directory and compiled there; the real oracle is never modified.
This shows the pins are sharp enough to catch a dropped term, a wrong sign, a
wrong index or a transposed step anywhere on the path."""
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
import oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "sv_oracle.c")

MUTANTS = {
    "temperature_after_log_softmax": (
        "s += exp((widen(base, is_bf16, off + (size_t)v) - M) / T);\n    *lse = M / T + log(s);",
        "s += exp(widen(base, is_bf16, off + (size_t)v) - M);\n    *lse = (M + log(s)) / T;"),
    "residual_sign_flipped": ("wbuf[v] = fmax(0.0, p - q);", "wbuf[v] = fmax(0.0, q - p);"),
    "residual_not_clamped": ("wbuf[v] = fmax(0.0, p - q);", "wbuf[v] = p - q;"),
    "linear_uniform_in_log_test": ("double lu = log((double)u_acc[j]);", "double lu = (double)u_acc[j];"),
    "gather_without_temperature": ("/ T - lse_t[j];", "- lse_t[j];"),
    "residual_from_next_position": (
        "double p = exp(widen(tgt, is_bf16, trow0 + (size_t)n * V + v) / T - lse_t[n]);",
        "double p = exp(widen(tgt, is_bf16, trow0 + (size_t)(n + 1) * V + v) / T - lse_t[n + 1]);"),
    "bonus_from_wrong_row": (
        "trow0 + (size_t)gamma * V + v) / T - lse_t[gamma]);",
        "trow0 + (size_t)(gamma - 1) * V + v) / T - lse_t[gamma - 1]);"),
    "greedy_last_argmax": ("if (l > best) { best = l; arg = v; }", "if (l >= best) { best = l; arg = v; }"),
    "scan_past_first_rejection": ("if (!(lu < delta)) { n = j; break; }", "if (!(lu < delta)) { n = j; }"),
    "cdf_not_scaled_by_total": ("double target = u * S;", "double target = u;"),
    "residual_fallback_removed": ("if (!(S >= ORACLE_RESIDUAL_MIN)) {", "if (0) {"),
    "residual_fallback_draws_from_q": (
        "                wbuf[v] = exp(widen(tgt, is_bf16, trow0 + (size_t)n * V + v) / T - lse_t[n]);",
        "                wbuf[v] = exp(widen(dft, is_bf16, drow0 + (size_t)n * V + v) / T - lse_d[n]);"),
    "residual_fallback_next_row": (
        "                wbuf[v] = exp(widen(tgt, is_bf16, trow0 + (size_t)n * V + v) / T - lse_t[n]);",
        "                wbuf[v] = exp(widen(tgt, is_bf16, trow0 + (size_t)(n + 1) * V + v) / T - lse_t[n + 1]);"),
    "residual_fallback_unflagged": ("st |= ST_RESID0;", ";"),
    "residual_threshold_zero": ("!(S >= ORACLE_RESIDUAL_MIN)", "!(S > 0.0)"),
    "accept_uniform_unchecked": ("if (!(u_acc[j] >= 0.0f && u_acc[j] < 1.0f)) st |= ST_UNIFORM;", ";"),
    "draft_normaliser_for_target": (
        "double lp = widen(tgt, is_bf16, trow0 + (size_t)j * V + (size_t)tok[j]) / T - lse_t[j];",
        "double lp = widen(tgt, is_bf16, trow0 + (size_t)j * V + (size_t)tok[j]) / T - lse_d[j];"),
}

# planted mistakes in the speculation-cache functions, caught by topf_pins
TOPF_MUTANTS = {
    "topf_ascending": ("if (x->w > y->w) return -1;\n    if (x->w < y->w) return 1;",
                       "if (x->w > y->w) return 1;\n    if (x->w < y->w) return -1;"),
    "topf_ties_larger_token_first": ("return (x->v > y->v) - (x->v < y->v);", "return (x->v < y->v) - (x->v > y->v);"),
    "topf_residual_not_clamped": ("buf[v].w = n < gamma ? fmax(0.0, pt - qd) : pt;", "buf[v].w = n < gamma ? pt - qd : pt;"),
    "topf_no_vanished_fallback": ("if (n < gamma && !(ORACLE_RESIDUAL_MIN <= S)) {", "if (0) {"),
    "topf_unnormalised": ("out_p[off + s] = buf[s].w / S;", "out_p[off + s] = buf[s].w;"),
    "topf_keeps_zero_weights": ("if (!(buf[s].w > 0.0)) break;", ";"),
    "fanout_uniform": ("const double P = n < gamma ? pow(alpha, n) * (1.0 - alpha) : pow(alpha, gamma);",
                       "const double P = 1.0 / (double)(gamma + 1);"),
    "fanout_remainder_to_last": ("if (rem > br) { br = rem; best = n; }", "if (rem >= br) { br = rem; best = n; }"),
    "lookup_wrong_outcome_slots": ("for (int s = off[n]; s < off[n + 1]; ++s)", "for (int s = 0; s < Ftot; ++s)"),
}

# planted mistakes in the draft-selection bandit, caught by bandit_pins
BANDIT_MUTANTS = {
    "bandit_reward_not_per_draft": ("const double reward = (double)acc / ((double)B * (double)gamma);",
                                    "const double reward = (double)acc / (double)B;"),
    "bandit_ucb_half_bonus": ("score = R[k] / N[k] + sqrt(2.0 * log(*t) / N[k]);",
                              "score = R[k] / N[k] + sqrt(log(*t) / N[k]);"),
    "bandit_ties_to_larger_arm": ("if (score > best) { best = score; pick = k; }",
                                  "if (score >= best) { best = score; pick = k; }"),
    "bandit_no_exploration_first": ("if (N[k] == 0.0) { pick = k; break; }", ";"),
    "bandit_thompson_narrow": ("score = R[k] / N[k] + z / sqrt(N[k] + 1.0);", "score = R[k] / N[k] + z / (N[k] + 1.0);"),
    "bandit_beta_no_prior": ("const double m = (R[k] + 1.0) / (N[k] + 2.0);", "const double m = R[k] / N[k];"),
    "bandit_beta_variance_n1": ("score = m + z * sqrt(m * (1.0 - m) / (N[k] + 3.0));",
                                "score = m + z * sqrt(m * (1.0 - m) / (N[k] + 1.0));"),
    "bandit_reward_to_arm0": ("N[*arm] += 1.0;\n        R[*arm] += reward;", "N[*arm] += 1.0;\n        R[0] += reward;"),
}

TREE_MUTANTS = {
    "tree_residual_sign": ("wbuf[v] = fmax(0.0, P - q);", "wbuf[v] = fmax(0.0, q - P);"),
    "tree_later_tests_use_p": ("const double lp = level == 0 ?", "const double lp = 1 ?"),
    "tree_residual_never_applied": ("if (S < ORACLE_RESIDUAL_MIN || S != S) {", "if (1) {"),
    "tree_keep_ignored": ("in[i] = in[par[i]] && (keep == NULL || keep[i] != 0);", "in[i] = in[par[i]];"),
    "tree_parent_off_by_one": ("if (par[i] < 0 || par[i] >= i) { st |= ST_TREE;", "if (par[i] < 0 || par[i] > i) { st |= ST_TREE;"),
    "tree_leaf_draft_row_read": ("if (first >= 0) {\n                if (!row_lse(dft", "if (first >= -1) {\n                if (!row_lse(dft"),
    "tree_greedy_inverted": ("if (tok[i] == a) { next = i; break; }", "if (tok[i] != a) { next = i; break; }"),
    "tree_fallback_not_flagged": ("st = st | ST_RESID0; /* the residual vanished: P stays */", "; /* P stays */"),
    "prune_child_row": ("const size_t row = (o + (size_t)c) * (size_t)V;", "const size_t row = (o + (size_t)i) * (size_t)V;"),
    # (keep[i] without keep[parent] is an equivalent mutant: log q <= 0, so a path's
    # cumulative log-probability never rises and a pruned parent's children fall below
    # the threshold too)
    "prune_not_cumulative": ("out_cum[o + i] = out_cum[o + c] + lq;", "out_cum[o + i] = lq;"),
}

LOWRANK_MUTANTS = {
    "lowrank_truncates": ("r = ldexp(nearbyint(ldexp(f, 8)), e - 8);", "r = ldexp(trunc(ldexp(f, 8)), e - 8);"),
    "gemm_b_transposed": ("bf16_value(B, (size_t)n * K + k)", "bf16_value(B, (size_t)k * N + n)"),
    "lowrank_lse_unrounded": ("s += exp((bf16_round(z[v]) - mx) / T);", "s += exp((z[v] - mx) / T);"),
    "lowrank_lse_no_temperature": ("out_lse[m] = mx / T + log(s);", "out_lse[m] = mx + log(s);"),
}

BANDIT_SIM_MUTANTS = {
    "sim_gap_from_first_arm": ("if (mu[k] > mu_max) mu_max = mu[k];", ";"),
    "sim_reward_draw_of_last_row": ("reward = (double)us[2 * K] < mu[arm] ? 1 : 0;",
                                    "reward = (double)us[-1] < mu[arm] ? 1 : 0;"),
    "sim_reward_inverted": ("reward = (double)us[2 * K] < mu[arm] ? 1 : 0;",
                            "reward = (double)us[2 * K] < mu[arm] ? 0 : 1;"),
    "sim_u2_from_u1": ("sv_oracle_bandit_step(&reward, 1, 1, &t, &arm, N, Rs, K, policy, us, us + K);",
                       "sv_oracle_bandit_step(&reward, 1, 1, &t, &arm, N, Rs, K, policy, us, us);"),
    "sim_regret_after_step": ("regret += mu_max - mu[arm];", ";"),
}


def _build_mutant(name, tmpdir):
    src = open(SRC).read()
    old, new = {**MUTANTS, **TOPF_MUTANTS, **BANDIT_MUTANTS, **BANDIT_SIM_MUTANTS, **TREE_MUTANTS, **LOWRANK_MUTANTS}[name]
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = os.path.join(tmpdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(tmpdir, f"lib_{name}.so")
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", so, path, "-lm"])
    return oracle.load_library(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    with tempfile.TemporaryDirectory() as d:
        lib = _build_mutant(name, d)

        def verify(*a, **k):
            return oracle.verify(*a, lib=lib, **k)

        caught = []
        for check in P.ALL_ORACLE_CHECKS:
            try:
                with np.errstate(all="ignore"):
                    check(verify)
            except Exception as e:  # noqa: BLE001 - any failure counts as caught
                caught.append((check.__name__, type(e).__name__))
                break
        if not caught:
            try:
                P.check_bonus_distribution(verify, min_samples=3000)
            except Exception as e:  # noqa: BLE001
                caught.append(("check_bonus_distribution", type(e).__name__))
        assert caught, f"planted mistake {name} passed every pin"


class _OracleWith:
    """The oracle's Python functions bound to a mutant library."""

    def __init__(self, lib):
        self.lib = lib

    def verify(self, *a, **k):
        return oracle.verify(*a, lib=self.lib, **k)

    def topf(self, *a, **k):
        return oracle.topf(*a, lib=self.lib, **k)

    def fanout(self, *a, **k):
        return oracle.fanout(*a, lib=self.lib, **k)

    def cache_lookup(self, *a, **k):
        return oracle.cache_lookup(*a, lib=self.lib, **k)

    def tree_verify(self, *a, **k):
        return oracle.tree_verify(*a, lib=self.lib, **k)

    def tree_prune(self, *a, **k):
        return oracle.tree_prune(*a, lib=self.lib, **k)

    def gemm_bf16(self, *a, **k):
        return oracle.gemm_bf16(*a, lib=self.lib, **k)

    def lowrank_head(self, *a, **k):
        return oracle.lowrank_head(*a, lib=self.lib, **k)


@pytest.mark.parametrize("name", sorted(TOPF_MUTANTS))
def test_topf_mutant_is_caught(name):
    import topf_pins as TP
    with tempfile.TemporaryDirectory() as d:
        O = _OracleWith(_build_mutant(name, d))
        caught = []
        for check in TP.ALL_TOPF_CHECKS:
            try:
                with np.errstate(all="ignore"):
                    check(O)
            except Exception as e:  # noqa: BLE001 - any failure counts as caught
                caught.append((check.__name__, type(e).__name__))
                break
        assert caught, f"planted mistake {name} passed every pin"


@pytest.mark.parametrize("name", sorted(BANDIT_MUTANTS))
def test_bandit_mutant_is_caught(name):
    import bandit_pins as BP
    with tempfile.TemporaryDirectory() as d:
        lib = _build_mutant(name, d)
        caught = []
        for check in BP.ALL_BANDIT_CHECKS:
            try:
                with np.errstate(all="ignore"):
                    check(lambda K, policy: oracle.Bandit(K, policy, lib=lib))
            except Exception as e:  # noqa: BLE001 - any failure counts as caught
                caught.append((check.__name__, type(e).__name__))
                break
        assert caught, f"planted mistake {name} passed every pin"


@pytest.mark.parametrize("name", sorted(BANDIT_SIM_MUTANTS))
def test_bandit_sim_mutant_is_caught(name):
    import bandit_pins as BP
    with tempfile.TemporaryDirectory() as d:
        lib = _build_mutant(name, d)
        clean = oracle.load_library(oracle.build())
        caught = []
        for check in BP.ALL_SIM_CHECKS:
            try:
                check(lambda mu, T, policy, U: oracle.bandit_simulate(mu, T, policy, U, lib=lib, with_state=True),
                      lambda K, policy: oracle.Bandit(K, policy, lib=clean))
            except Exception as e:  # noqa: BLE001 - any failure counts as caught
                caught.append((check.__name__, type(e).__name__))
                break
        assert caught, f"planted mistake {name} passed every pin"


@pytest.mark.parametrize("name", sorted(TREE_MUTANTS))
def test_tree_mutant_is_caught(name):
    import tree_pins as TP
    with tempfile.TemporaryDirectory() as d:
        O = _OracleWith(_build_mutant(name, d))
        caught = []
        for check in TP.ALL_TREE_CHECKS:
            try:
                with np.errstate(all="ignore"):
                    check(O)
            except Exception as e:  # noqa: BLE001 - any failure counts as caught
                caught.append((check.__name__, type(e).__name__))
                break
        assert caught, f"planted mistake {name} passed every pin"


@pytest.mark.parametrize("name", sorted(LOWRANK_MUTANTS))
def test_lowrank_mutant_is_caught(name):
    import lowrank_pins as LP
    with tempfile.TemporaryDirectory() as d:
        O = _OracleWith(_build_mutant(name, d))
        caught = []
        for check in LP.ALL_LOWRANK_CHECKS:
            try:
                with np.errstate(all="ignore"):
                    check(O)
            except Exception as e:  # noqa: BLE001 - any failure counts as caught
                caught.append((check.__name__, type(e).__name__))
                break
        assert caught, f"planted mistake {name} passed every pin"
