"""Exact law of one speculative-sampling verification step, by enumeration.

Written from the mathematics of speculative sampling, independently of the
oracle: for tiny vocabularies every draft sequence x (probability prod q_j(x_j))
is enumerated and the uniforms are integrated out analytically:

  * position j is accepted with probability min(1, p_j(x_j) / q_j(x_j));
  * after a rejection at m the extra token is k with probability
    max(0, p_m(k) - q_m(k)) / sum_v max(0, p_m(v) - q_m(v));
  * after gamma acceptances the bonus token is k with probability p_gamma(k).

Works on ``fractions.Fraction`` (exact) or floats.  Used to pin the oracle and
to state the pages' distribution-preservation property (FlashSpec, Metodologia 2
"Garantia Teorica" and Teorema 1) as an exact identity.
"""
from __future__ import annotations

import itertools
from collections import defaultdict
from fractions import Fraction


def outcome_law(p, q):
    """Return {(n, tokens tuple of length n+1): probability}.

    p: gamma+1 distributions (lists) over V tokens; q: gamma distributions."""
    gamma = len(q)
    V = len(p[0])
    zero = p[0][0] * 0
    law = defaultdict(lambda: zero)
    for x in itertools.product(range(V), repeat=gamma):
        w = zero + 1
        for j in range(gamma):
            w = w * q[j][x[j]]
        if w == 0:
            continue
        still = zero + 1  # probability that positions < m were all accepted
        for m in range(gamma):
            a = min(zero + 1, p[m][x[m]] / q[m][x[m]])
            reject = still * (1 - a)
            if reject > 0:
                r = [max(zero, p[m][v] - q[m][v]) for v in range(V)]
                S = sum(r, zero)
                for k in range(V):
                    if r[k] > 0:
                        law[(m, tuple(x[:m]) + (k,))] += w * reject * r[k] / S
            still = still * a
            if still == 0:
                break
        if still > 0:
            for k in range(V):
                if p[gamma][k] > 0:
                    law[(gamma, tuple(x) + (k,))] += w * still * p[gamma][k]
    return dict(law)


def closed_form_law(p, q):
    """P(n = m, y) = prod_{i<m} min(p_i, q_i)(y_i) * max(0, p_m - q_m)(y_m)   (m < gamma)
       P(n = gamma, y) = prod_{i<gamma} min(p_i, q_i)(y_i) * p_gamma(y_gamma)."""
    gamma = len(q)
    V = len(p[0])
    zero = p[0][0] * 0
    law = {}
    for m in range(gamma + 1):
        for y in itertools.product(range(V), repeat=m + 1):
            pr = zero + 1
            for i in range(m):
                pr = pr * min(p[i][y[i]], q[i][y[i]])
            last = p[m][y[m]] if m == gamma else max(zero, p[m][y[m]] - q[m][y[m]])
            pr = pr * last
            if pr > 0:
                law[(m, y)] = pr
    return law


def overlap(p_row, q_row):
    """beta = sum_v min(p_v, q_v): the acceptance probability of one position."""
    return sum((min(a, b) for a, b in zip(p_row, q_row)), p_row[0] * 0)


def random_rational_dist(rng, V, denom=64, allow_zero=True):
    """A random distribution with small-denominator rational masses."""
    while True:
        w = [int(rng.integers(0 if allow_zero else 1, denom)) for _ in range(V)]
        if sum(w) > 0:
            s = sum(w)
            return [Fraction(a, s) for a in w]


def to_float(law):
    return {k: float(v) for k, v in law.items()}


def position_marginals(law, gamma, V):
    """emit[j][v] = P(position j is emitted and equals v); reach[j] = P(n >= j)."""
    emit = [[0.0] * V for _ in range(gamma + 1)]
    for (n, y), pr in law.items():
        for j in range(n + 1):
            emit[j][y[j]] += float(pr)
    reach = [sum(row) for row in emit]
    return emit, reach
