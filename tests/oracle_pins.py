"""Checks that pin the CPU oracle to facts outside itself.

Each ``check_*`` takes a ``verify`` callable with the signature of
``oracle.verify`` and raises AssertionError on a violation.  The same battery
runs against the real oracle (tests/test_oracle_pins.py) and against copies of
the oracle with a planted mistake (tests/test_oracle_mutants.py), which must
each fail at least one check.

Every expected value here is computed independently of the oracle: closed
forms, ``math.fsum`` log-sum-exp, ``numpy.argmax`` / ``numpy.searchsorted``,
and the exact rational law of ``exact_law.py``.
"""
from __future__ import annotations

import itertools
import math
from fractions import Fraction

import numpy as np

import exact_law
from speculative_decoding_verification_84_b200 import workloads as W


# ----------------------------------------------------------------- independent helpers

def fsum_lse(row, T):
    """Textbook log-sum-exp of row/T with an exactly rounded sum (math.fsum)."""
    row = [float(x) for x in row]
    M = max(row)
    return M / T + math.log(math.fsum(math.exp((x - M) / T) for x in row))


def fsum_softmax(row, T):
    lse = fsum_lse(row, T)
    return np.array([math.exp(float(x) / T - lse) for x in row])


def _seq_batch(target, draft, tokens, T, ua, ur):
    return (np.ascontiguousarray(target, dtype=np.float32), np.ascontiguousarray(draft, dtype=np.float32),
            np.ascontiguousarray(tokens, dtype=np.int32), np.ascontiguousarray(T, dtype=np.float32),
            np.ascontiguousarray(ua, dtype=np.float32), np.ascontiguousarray(ur, dtype=np.float32))


# ----------------------------------------------------------------- log-normaliser

def check_lse_constant_rows(verify):
    """Constant logits c: lse = c/T + ln V exactly (up to one rounding)."""
    for V, c, T in [(1, 0.0, 1.0), (7, 2.5, 0.5), (32000, -3.25, 1.0), (64, 10.0, 3.0)]:
        gamma = 2
        tgt = np.full((1, gamma + 1, V), c, np.float32)
        dft = np.full((1, gamma, V), c, np.float32)
        r = verify(*_seq_batch(tgt, dft, np.zeros((1, gamma)), [T], np.full((1, gamma), 0.5), [0.5]))
        want = c / T + math.log(V)
        assert np.allclose(r.log_norm[0], want, rtol=0, atol=1e-12 * max(1.0, abs(want))), (V, c, T)


def check_lse_shift_invariance(verify):
    """lse(l + c) = lse(l) + c/T for an exactly representable shift."""
    rng = np.random.default_rng(5)
    V, gamma, T = 1000, 2, float(np.float32(0.7))
    base = (rng.integers(-64, 64, size=(1, gamma + 1, V)) / 16.0).astype(np.float32)
    d = (rng.integers(-64, 64, size=(1, gamma, V)) / 16.0).astype(np.float32)
    args = (np.zeros((1, gamma)), [T], np.full((1, gamma), 0.5), [0.5])
    r0 = verify(*_seq_batch(base, d, *args))
    r1 = verify(*_seq_batch(base + 8.0, d + 8.0, *args))
    assert np.allclose(r1.log_norm - r0.log_norm, 8.0 / T, rtol=0, atol=1e-11)


def check_lse_fsum(verify):
    """Per-row normaliser against math.fsum log-sum-exp on config c1 and c2 rows."""
    for name in ("c1", "c2"):
        w = W.make_workload(name, seqs=[0])
        r = verify(w.target, w.draft, w.draft_tokens, w.temperature, w.u_accept, w.u_resample,
                   bf16=(w.dtype == "bf16"))
        T = float(w.temperature[0])
        t64, d64 = w.logits_as_f64("target")[0], w.logits_as_f64("draft")[0]
        want = [fsum_lse(t64[j], T) for j in range(w.gamma + 1)] + \
               [fsum_lse(d64[j], T) for j in range(w.gamma)]
        assert np.allclose(r.log_norm[0], want, rtol=0, atol=1e-10), name


def check_masked_vocab(verify):
    """-inf logits have zero probability: never emitted, normaliser of the rest."""
    V, gamma, T = 6, 1, 1.0
    row = np.array([-np.inf, 1.0, -np.inf, 2.0, -np.inf, 0.5], np.float32)
    tgt = np.tile(row, (200, gamma + 1, 1))
    dft = np.tile(np.array([-np.inf, 2.0, -np.inf, 1.0, -np.inf, 0.5], np.float32), (200, gamma, 1))
    rng = np.random.default_rng(1)
    toks = rng.choice([1, 3, 5], size=(200, gamma))
    r = verify(*_seq_batch(tgt, dft, toks, np.full(200, T), W.draw_uniforms(rng, (200, gamma)),
                           W.draw_uniforms(rng, (200,))))
    assert (r.row_status == 0).all()
    emitted = r.out_tokens[r.out_tokens >= 0]
    assert set(np.unique(emitted)) <= {1, 3, 5}
    assert abs(r.log_norm[0, 0] - fsum_lse([1.0, 2.0, 0.5], T)) < 1e-12


# ----------------------------------------------------------------- greedy

def check_greedy_argmax(verify):
    """T = 0: accept while x_j is the first argmax (numpy.argmax); ties -> lowest index."""
    rng = np.random.default_rng(11)
    B, gamma, V = 64, 3, 9
    tgt = rng.integers(-3, 3, size=(B, gamma + 1, V)).astype(np.float32)  # many ties
    dft = rng.standard_normal((B, gamma, V)).astype(np.float32)
    am = np.argmax(tgt, axis=-1)
    toks = am[:, :gamma].copy()
    for b in range(B):                      # break the draft at a random position
        k = b % (gamma + 1)
        if k < gamma:
            toks[b, k] = (am[b, k] + 1 + b % (V - 1)) % V
    r = verify(*_seq_batch(tgt, dft, toks, np.zeros(B), np.full((B, gamma), 0.5), np.full(B, 0.5)))
    for b in range(B):
        n = next((j for j in range(gamma) if toks[b, j] != am[b, j]), gamma)
        want = list(toks[b, :n]) + [am[b, n]] + [-1] * (gamma - n)
        assert r.n_accepted[b] == n and list(r.out_tokens[b]) == want, b


# ----------------------------------------------------------------- accept test

def check_accept_boundary(verify):
    """log u < log p - log q: u just below p/q accepts, just above rejects."""
    rng = np.random.default_rng(3)
    B, gamma, V, T = 40, 1, 50, float(np.float32(0.8))
    tgt = rng.standard_normal((B, gamma + 1, V)).astype(np.float32) * 2
    dft = (tgt[:, :gamma] + rng.standard_normal((B, gamma, V)) * 1.5).astype(np.float32)
    toks = rng.integers(0, V, size=(B, gamma))
    ua = np.empty((B, gamma), np.float32)
    expect = np.empty(B, bool)
    for b in range(B):
        p = fsum_softmax(tgt[b, 0], T)[toks[b, 0]]
        q = fsum_softmax(dft[b, 0], T)[toks[b, 0]]
        ratio = p / q
        while ratio >= 1.0:                              # need a boundary inside (0, 1)
            toks[b, 0] = (toks[b, 0] + 1) % V
            p = fsum_softmax(tgt[b, 0], T)[toks[b, 0]]
            q = fsum_softmax(dft[b, 0], T)[toks[b, 0]]
            ratio = p / q
        below = np.nextafter(np.float32(ratio), np.float32(0))
        above = np.nextafter(np.float32(ratio), np.float32(1))
        below = np.nextafter(below, np.float32(0))
        above = np.nextafter(above, np.float32(1))
        ua[b, 0] = below if b % 2 == 0 else above
        expect[b] = b % 2 == 0
    r = verify(*_seq_batch(tgt, dft, toks, np.full(B, T), ua, np.full(B, 0.5)))
    assert ((r.n_accepted == 1) == expect).all()


# ----------------------------------------------------------------- inverse CDF

def check_inverse_cdf_searchsorted(verify):
    """The extra token equals numpy.searchsorted(cumsum(w), u*S, side='right')."""
    for name in ("c2", "c3"):
        w = W.make_workload(name, seqs=range(8))
        r = verify(w.target, w.draft, w.draft_tokens, w.temperature, w.u_accept, w.u_resample,
                   bf16=(w.dtype == "bf16"))
        t64, d64 = w.logits_as_f64("target"), w.logits_as_f64("draft")
        for b in range(w.B):
            if r.cdf_gap[b] < 1e-9:
                continue
            T = float(w.temperature[b])
            n = int(r.n_accepted[b])
            p = np.exp(t64[b, n] / T - fsum_lse(t64[b, n], T))
            if n < w.gamma:
                q = np.exp(d64[b, n] / T - fsum_lse(d64[b, n], T))
                wts = np.maximum(0.0, p - q)
            else:
                wts = p
            C = np.cumsum(wts)
            k = int(np.searchsorted(C, float(w.u_resample[b]) * C[-1], side="right"))
            assert r.out_tokens[b, n] == k, (name, b)


# ----------------------------------------------------------------- exact law (pure maths)

def check_exact_law_identities():
    """Enumeration over drafts and uniforms equals the closed-form law, exactly."""
    rng = np.random.default_rng(17)
    for gamma, V in [(1, 2), (1, 5), (2, 3), (3, 3), (2, 4), (3, 2)]:
        for _ in range(3):
            p = [exact_law.random_rational_dist(rng, V) for _ in range(gamma + 1)]
            q = [exact_law.random_rational_dist(rng, V) for _ in range(gamma)]
            law = exact_law.outcome_law(p, q)
            assert law == exact_law.closed_form_law(p, q)
            assert sum(law.values()) == 1
            # distribution preservation: emitted token at j is p_j given emission,
            # and P(n >= j) = prod_{i<j} beta_i
            emit = [[Fraction(0)] * V for _ in range(gamma + 1)]
            for (n, y), pr in law.items():
                for j in range(n + 1):
                    emit[j][y[j]] += pr
            reach = Fraction(1)
            for j in range(gamma + 1):
                assert emit[j] == [reach * p[j][v] for v in range(V)]
                if j < gamma:
                    reach *= exact_law.overlap(p[j], q[j])


def check_oracle_partition(verify):
    """The oracle's map on interior points of every analytic outcome cell.

    For each draft sequence x and each outcome (first rejection m, token k), the
    uniforms are placed strictly inside that cell: u_i = a_i/2 for i < m (accept),
    u_m = (1 + a_m)/2 (reject), u_res at the centre of bin k.  The oracle must
    return exactly (m, x[:m] + [k])."""
    rng = np.random.default_rng(23)
    for gamma, V, T in [(1, 4, 1.0), (2, 3, float(np.float32(0.6))), (3, 3, float(np.float32(1.3))),
                        (2, 6, 1.0)]:
        tgt1 = (rng.standard_normal((gamma + 1, V)) * 1.5).astype(np.float32)
        dft1 = (rng.standard_normal((gamma, V)) * 1.5).astype(np.float32)
        p = [fsum_softmax(tgt1[j], T) for j in range(gamma + 1)]
        q = [fsum_softmax(dft1[j], T) for j in range(gamma)]
        rows, want = [], []
        for x in itertools.product(range(V), repeat=gamma):
            a = [min(1.0, p[j][x[j]] / q[j][x[j]]) for j in range(gamma)]
            for m in range(gamma + 1):
                if any(a[i] < 1e-5 for i in range(m)):
                    continue
                if m < gamma and a[m] > 1 - 1e-5:
                    continue
                wts = np.maximum(0.0, p[m] - q[m]) if m < gamma else p[gamma]
                C = np.concatenate([[0.0], np.cumsum(wts)])
                S = C[-1]
                for k in range(V):
                    if wts[k] / S < 1e-5:
                        continue
                    ua = [a[i] / 2 for i in range(m)]
                    if m < gamma:
                        ua += [(1 + a[m]) / 2] + [0.5] * (gamma - m - 1)
                    rows.append((x, ua, (C[k] + C[k + 1]) / 2 / S))
                    want.append((m, list(x[:m]) + [k] + [-1] * (gamma - m)))
        Bn = len(rows)
        toks = np.array([r_[0] for r_ in rows], np.int32).reshape(Bn, gamma)
        ua = np.array([r_[1] for r_ in rows], np.float32).reshape(Bn, gamma)
        ur = np.array([r_[2] for r_ in rows], np.float32)
        res = verify(*_seq_batch(np.tile(tgt1, (Bn, 1, 1)), np.tile(dft1, (Bn, 1, 1)), toks,
                                 np.full(Bn, T), ua, ur))
        for i, (m, tk) in enumerate(want):
            assert res.n_accepted[i] == m and list(res.out_tokens[i]) == tk, (gamma, V, i)


# ----------------------------------------------------------------- Monte Carlo law

def _chi2_pvalue(counts, probs):
    from scipy import stats
    n = counts.sum()
    exp_ = probs * n
    order = np.argsort(exp_)
    # merge the smallest expected bins until every bin expects >= 5
    c_m, e_m = [], []
    acc_c = acc_e = 0.0
    for i in order:
        acc_c += counts[i]
        acc_e += exp_[i]
        if acc_e >= 5:
            c_m.append(acc_c)
            e_m.append(acc_e)
            acc_c = acc_e = 0.0
    if acc_e > 0:
        c_m[-1] += acc_c
        e_m[-1] += acc_e
    c_m, e_m = np.array(c_m), np.array(e_m)
    e_m *= c_m.sum() / e_m.sum()
    return stats.chisquare(c_m, e_m).pvalue


def _ks_stat(counts, probs):
    n = counts.sum()
    return np.max(np.abs(np.cumsum(counts) / n - np.cumsum(probs))), n


def distribution_trials(verify, tgt1, dft1, T, n_rows, seed):
    """Run n_rows independent verifications of one (target, draft) pattern, drafts ~ q."""
    gamma = dft1.shape[0]
    V = dft1.shape[1]
    rng = np.random.default_rng(seed)
    gu = np.clip(rng.random((n_rows, gamma, V)), 1e-300, 1 - 2.0 ** -53)
    toks = np.argmax(dft1.astype(np.float64)[None] / T - np.log(-np.log(gu)), axis=-1)
    r = verify(*_seq_batch(np.broadcast_to(tgt1, (n_rows,) + tgt1.shape),
                           np.broadcast_to(dft1, (n_rows,) + dft1.shape), toks,
                           np.full(n_rows, T), W.draw_uniforms(rng, (n_rows, gamma)),
                           W.draw_uniforms(rng, (n_rows,))))
    return r


def check_distribution(verify, positions=(0, 1, 2), min_samples=10_000, patterns=(0, 1, 2),
                       alpha=0.01):
    """Emitted token at position j, given that j is emitted, follows p_j (chi-square and
    KS at significance alpha over >= min_samples trials); P(n >= j) = prod beta_i."""
    for pat in patterns:
        w = W.make_workload("c5", seqs=[0], pattern=pat)
        tgt1, dft1, T = w.target[0], w.draft[0], 1.0
        gamma, V = w.gamma, w.V
        p = [fsum_softmax(tgt1[j], T) for j in range(gamma + 1)]
        q = [fsum_softmax(dft1[j], T) for j in range(gamma)]
        beta = [float(np.minimum(p[j], q[j]).sum()) for j in range(gamma)]
        counts = {j: np.zeros(V) for j in positions}
        total_rows = 0
        reach = np.zeros(gamma + 1)
        it = 0
        while min(counts[j].sum() for j in positions) < min_samples:
            r = distribution_trials(verify, tgt1, dft1, T, 16384, seed=1000 * pat + it)
            it += 1
            total_rows += 16384
            for j in range(gamma + 1):
                reach[j] += (r.n_accepted >= j).sum()
            for j in positions:
                sel = r.n_accepted >= j
                counts[j] += np.bincount(r.out_tokens[sel, j], minlength=V)
            assert it < 40
        for j in positions:
            pv = _chi2_pvalue(counts[j], p[j])
            D, n = _ks_stat(counts[j], p[j])
            assert pv > alpha, (pat, j, pv)
            assert D < 1.628 / math.sqrt(n), (pat, j, D)
        prob = 1.0
        for j in range(gamma + 1):
            sd = math.sqrt(total_rows * prob * (1 - prob)) + 1e-9
            assert abs(reach[j] - total_rows * prob) < 4 * sd + 1e-9, (pat, j, reach[j], prob)
            if j < gamma:
                prob *= beta[j]


def check_bonus_distribution(verify, min_samples=10_000, alpha=0.01):
    """All-accepted rows: the bonus token follows p_gamma (high-overlap pattern)."""
    rng = np.random.default_rng(77)
    gamma, V, T = 4, 64, 1.0
    tgt1 = (rng.standard_normal((gamma + 1, V)) * 1.5).astype(np.float32)
    dft1 = (tgt1[:gamma] + rng.standard_normal((gamma, V)) * 0.15).astype(np.float32)
    p = fsum_softmax(tgt1[gamma], T)
    counts = np.zeros(V)
    it = 0
    while counts.sum() < min_samples:
        r = distribution_trials(verify, tgt1, dft1, T, 16384, seed=5000 + it)
        it += 1
        sel = r.n_accepted == gamma
        counts += np.bincount(r.out_tokens[sel, gamma], minlength=V)
        assert it < 20
    assert _chi2_pvalue(counts, p) > alpha
    D, n = _ks_stat(counts, p)
    assert D < 1.628 / math.sqrt(n)


# ----------------------------------------------------------------- vanished residual

RESIDUAL_MIN = 2.0 ** -18   # the contract's threshold: a smaller residual mass counts as vanished


def vanished_residual_cases(V, seed=41):
    """Rows whose residual at position 0 vanishes, with the uniforms to use.

    Target and draft row 0 are equal except at one token x, and the draft token
    at position 0 is x, whose log ratio is about -0.75 or -1, so u_accept = 0.75
    rejects it (log 0.75 = -0.29).
      (a) both logits at x sit ~100 below the rest: the normalisers of the two
          rows agree to far below rounding, so p_v = q_v for v != x and p_x < q_x:
          the residual mass S is 0;
      (b) p_0 ~ 1.3e-6 and the draft raises logit 0 by 1 (x = 0): S = q_0 - p_0
          ~ 2.2e-6, still more than 1e-6 below 2^-18.  u_resample is placed
          1.6e-6 above p_0, inside q's first bin but past p's, so a draw from
          q instead of p would return token 0.
    Returns a list of (lt_row0, ld_row0, x, u_resample) in float32."""
    rng = np.random.default_rng(seed)
    base = (rng.standard_normal(V) * 1.5).astype(np.float32)
    out = []
    x = min(7, V - 1)
    lt = base.copy(); lt[x] = np.float32(-100.0)
    ld = base.copy(); ld[x] = np.float32(-99.25)
    for u in (0.3, 0.6, 0.95):
        out.append((lt, ld, x, np.float32(u)))
    lse_rest = fsum_lse(base[1:], 1.0)
    lt = base.copy(); lt[0] = np.float32(lse_rest + math.log(1.3e-6))
    ld = lt.copy(); ld[0] = np.float32(float(lt[0]) + 1.0)
    p0 = float(fsum_softmax(lt, 1.0)[0])
    for u in (p0 + 1.6e-6, 0.4, 0.9):
        out.append((lt, ld, 0, np.float32(u)))
    return out


def check_residual_vanished(verify):
    """Residual mass below 2^-18 after a rejection: status 8, n = 0, and the token is
    numpy.searchsorted(cumsum(p_0), u * sum(p_0), 'right') with p_0 from math.fsum
    (Speculative Speculative Decoding, Desafios 2, "Amostragem Saguaro": the
    residual; the fallback is the library's reading for a residual that vanished)."""
    V, gamma, T = 40, 2, 1.0
    rng = np.random.default_rng(43)
    cases = vanished_residual_cases(V)
    B = len(cases)
    tgt = (rng.standard_normal((B, gamma + 1, V)) * 1.5).astype(np.float32)
    dft = (rng.standard_normal((B, gamma, V)) * 1.5).astype(np.float32)
    toks = rng.integers(0, V, size=(B, gamma))
    ur = np.empty(B, np.float32)
    for i, (lt, ld, x, u) in enumerate(cases):
        tgt[i, 0], dft[i, 0], toks[i, 0], ur[i] = lt, ld, x, u
    ua = np.full((B, gamma), 0.75, np.float32)
    r = verify(*_seq_batch(tgt, dft, toks, np.full(B, T), ua, ur))
    for i, (lt, ld, x, u) in enumerate(cases):
        p = fsum_softmax(lt.astype(np.float64), T)
        q = fsum_softmax(ld.astype(np.float64), T)
        S = math.fsum(np.maximum(0.0, p - q))
        assert S < RESIDUAL_MIN - 1e-6, (i, S)          # the construction itself
        C = np.cumsum(p)
        target = float(u) * C[-1]
        k = int(np.searchsorted(C, target, side="right"))
        lo = C[k - 1] if k > 0 else 0.0
        assert min(target - lo, C[k] - target) > 1e-6, i  # a clean draw, not a near tie
        assert r.row_status[i] == 8, (i, r.row_status[i])
        assert r.n_accepted[i] == 0, i
        assert list(r.out_tokens[i]) == [k] + [-1] * gamma, (i, k, r.out_tokens[i])
        assert r.cdf_gap[i] >= 1e-6, (i, r.cdf_gap[i])


# ----------------------------------------------------------------- contract edges

def check_status_edges(verify):
    """Invalid temperature -> 4; token out of range -> 1; NaN/+inf/all -inf row -> 2;
    a uniform outside [0, 1) or NaN -> 16 (T > 0 only: a greedy sequence reads none)."""
    V, gamma = 16, 2
    rng = np.random.default_rng(2)
    base_t = rng.standard_normal((gamma + 1, V)).astype(np.float32)
    base_d = rng.standard_normal((gamma, V)).astype(np.float32)
    ok_u = ([0.5, 0.5], 0.5)
    cases = []
    for T in (-1.0, np.nan, np.inf, 1e-7):
        cases.append((base_t, base_d, [1, 2], T, 4, ok_u))
    cases.append((base_t, base_d, [1, V], 1.0, 1, ok_u))
    cases.append((base_t, base_d, [-1, 0], 0.0, 1, ok_u))
    bad = base_t.copy(); bad[1, 3] = np.nan
    cases.append((bad, base_d, [1, 2], 1.0, 2, ok_u))
    cases.append((bad, base_d, [1, 2], 0.0, 2, ok_u))
    bad = base_d.copy(); bad[0, :] = -np.inf
    cases.append((base_t, bad, [1, 2], 1.0, 2, ok_u))
    cases.append((base_t, bad, [1, 2], 0.0, 0, ok_u))   # greedy never reads draft rows
    bad = base_t.copy(); bad[2, 5] = np.inf
    cases.append((bad, base_d, [1, 2], 1.0, 2, ok_u))
    for ua, ur in (([1.0, 0.5], 0.5), ([np.nan, 0.5], 0.5), ([0.5, -0.25], 0.5), ([0.5, 0.5], 1.0),
                   ([0.5, 0.5], np.nan), ([0.5, 0.5], np.inf)):
        cases.append((base_t, base_d, [1, 2], 1.0, 16, (ua, ur)))
    cases.append((base_t, base_d, [1, V], 1.0, 17, ([2.0, 0.5], 0.5)))
    cases.append((base_t, base_d, [1, 2], 1.0, 0, ([0.0, 0.0], 0.0)))   # 0 is in [0, 1)
    cases.append((base_t, base_d, [1, 2], 0.0, 0, ([1.0, np.nan], 7.0)))  # greedy reads no uniform
    for tg, dg, tk, T, st, (ua, ur) in cases:
        r = verify(*_seq_batch(tg[None], dg[None], [tk], [T], [ua], [ur]))
        assert r.row_status[0] == st, (T, tk, st, r.row_status[0], ua, ur)
        if st & 23:
            assert r.n_accepted[0] == 0 and (r.out_tokens[0] == -1).all()
        if st == 4 or T == 0.0:
            assert np.isnan(r.log_norm[0]).all()


def check_output_invariants(verify):
    """On random shapes: n in [0, gamma]; accepted prefix = drafts; extra token has
    positive weight under the distribution it was drawn from; -1 afterwards."""
    rng = np.random.default_rng(31)
    for B, gamma, V, dt in [(5, 1, 1, "f32"), (7, 3, 13, "bf16"), (3, 6, 257, "f32"), (9, 2, 33, "bf16")]:
        T = rng.choice([0.0, 0.5, 1.0, 2.0], size=B)
        w = W.make_random(B, gamma, V, dt, seed=int(rng.integers(1 << 30)), T=T)
        r = verify(w.target, w.draft, w.draft_tokens, w.temperature, w.u_accept, w.u_resample,
                   bf16=(dt == "bf16"))
        t64, d64 = w.logits_as_f64("target"), w.logits_as_f64("draft")
        for b in range(B):
            n = int(r.n_accepted[b])
            assert 0 <= n <= gamma
            assert list(r.out_tokens[b, :n]) == list(w.draft_tokens[b, :n])
            assert (r.out_tokens[b, n + 1:] == -1).all()
            k = int(r.out_tokens[b, n])
            Tb = float(w.temperature[b])
            if Tb == 0.0:
                assert k == int(np.argmax(t64[b, n]))
            else:
                p = fsum_softmax(t64[b, n], Tb)
                if n < gamma:
                    q = fsum_softmax(d64[b, n], Tb)
                    assert p[k] > q[k] or r.row_status[b] & 8
                else:
                    assert p[k] > 0


ALL_ORACLE_CHECKS = [
    check_lse_constant_rows, check_lse_shift_invariance, check_lse_fsum, check_masked_vocab,
    check_greedy_argmax, check_accept_boundary, check_inverse_cdf_searchsorted,
    check_residual_vanished, check_oracle_partition, check_status_edges, check_output_invariants,
]
