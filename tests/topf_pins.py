"""Pins of the oracle's speculation-cache functions (fan-out, top-F per outcome,
cache lookup), each against something other than the oracle itself: hand-worked
cases, numpy sorts of independently computed probabilities, and properties of
the definitions.  Every check takes the oracle module (or a stand-in with the
same functions, for planted mistakes) as its argument.

The passages: Speculative Speculative Decoding, Metodologia 2 ("Conceito
Central": the outcome is the number accepted plus one token, the cache holds
speculations for likely outcomes) and Desafios 1 (geometric fan-out over the
accepted lengths) and 2 (the extra token after a rejection follows the
residual, whose mass Saguaro sampling moves onto the cached top-F tokens)."""
from __future__ import annotations

import math

import numpy as np


def _softmax64(row, T):
    z = row.astype(np.float64) / T
    z = z - z.max()
    e = np.exp(z)
    return e / e.sum()


def expected_topf(target, draft, T, F, residual_min=2.0 ** -18):
    """Independent restatement with numpy (float64): per outcome n the residual
    max(0, p_n - q_n) (p_n if its mass is below residual_min) or p_gamma, its F_n
    largest probabilities, ties broken by the smaller token."""
    B, g1, V = target.shape
    gamma = g1 - 1
    Ft = int(np.sum(F))
    tok = np.full((B, Ft), -1, np.int32)
    prob = np.zeros((B, Ft))
    for b in range(B):
        off = 0
        for n in range(gamma + 1):
            if T[b] == 0:
                if F[n] > 0:
                    tok[b, off] = int(np.argmax(target[b, n]))
                    prob[b, off] = 1.0
                off += F[n]
                continue
            p = _softmax64(target[b, n], T[b])
            if n < gamma:
                w = np.maximum(0.0, p - _softmax64(draft[b, n], T[b]))
                if not w.sum() >= residual_min:
                    w = p
            else:
                w = p
            order = np.lexsort((np.arange(V), -w))  # by -w, then by token
            k = 0
            for v in order[:F[n]]:
                if w[v] > 0:
                    tok[b, off + k] = v
                    prob[b, off + k] = w[v] / w.sum()
                    k += 1
            off += F[n]
    return tok, prob


def check_fanout_closed_forms(O):
    # alpha = 1/2, gamma = 3: P = (1/2, 1/4, 1/8, 1/8), times 16 is exact
    assert O.fanout(0.5, 3, 16).tolist() == [8, 4, 2, 2]
    # alpha = 0: every outcome is n = 0; alpha = 1: every outcome is n = gamma
    assert O.fanout(0.0, 3, 5).tolist() == [5, 0, 0, 0]
    assert O.fanout(1.0, 3, 5).tolist() == [0, 0, 0, 5]
    # alpha = 0.7, gamma = 5, budget 64: 64 * P = 19.2, 13.44, 9.408, 6.5856,
    # 4.60992, 10.75648; floors 19, 13, 9, 6, 4, 10 (61); the 3 left go to the
    # largest remainders .75648 (n=5), .60992 (n=4), .5856 (n=3)
    assert O.fanout(0.7, 5, 64).tolist() == [19, 13, 9, 7, 5, 11]
    # alpha = 1/2, gamma = 1: P = (1/2, 1/2), 3 slots -> 1.5 each; the slot left
    # over goes to the smaller n on the tie
    assert O.fanout(0.5, 1, 3).tolist() == [2, 1]
    for alpha in (0.1, 0.33, 0.8, 0.95):
        for gamma in (1, 4, 8):
            for budget in (0, 1, 7, 100):
                F = O.fanout(alpha, gamma, budget)
                assert F.sum() == budget and (F >= 0).all()
                P = [alpha ** n * (1 - alpha) for n in range(gamma)] + [alpha ** gamma]
                # every F_n is its share rounded down or up
                for n in range(gamma + 1):
                    assert math.floor(budget * P[n]) <= F[n] <= math.floor(budget * P[n]) + 1


def check_topf_hand_case(O):
    """V = 4, T = 1: target row 0 has p = (0.1, 0.2, 0.3, 0.4) (logits log 1..4),
    draft row 0 is uniform (q = 0.25): max(0, p - q) = (0, 0, 0.05, 0.15), S = 0.2,
    so the residual is (0, 0, 0.25, 0.75): top-3 = tokens 3, 2 and an empty slot.
    The bonus row is uniform: top-2 = tokens 0, 1 (ties: smaller token first)."""
    t = np.log(np.array([[[1, 2, 3, 4], [1, 1, 1, 1]]], np.float64)).astype(np.float32)
    d = np.zeros((1, 1, 4), np.float32)
    tok, prob = O.topf(t, d, np.array([1.0], np.float32), [3, 2])
    assert tok.tolist() == [[3, 2, -1, 0, 1]]
    assert np.allclose(prob, [[0.75, 0.25, 0.0, 0.25, 0.25]], atol=1e-6)


def check_topf_numpy(O):
    rng = np.random.default_rng(5)
    for V, gamma, dt in ((50, 3, "f32"), (97, 2, "f32"), (64, 4, "bf16")):
        B = 7
        t = (rng.standard_normal((B, gamma + 1, V)) * 2).astype(np.float32)
        d = (t[:, :gamma] + rng.standard_normal((B, gamma, V))).astype(np.float32)
        T = np.array([1.0, 0.7, 1.3, 0.0, 1.0, 2.0, 0.5][:B], np.float32)
        F = [3, 5, 1, 0, 2, 4][: gamma + 1]
        if dt == "bf16":
            tb = (t.view(np.uint32) >> 16).astype(np.uint16)
            db = (d.view(np.uint32) >> 16).astype(np.uint16)
            tf = (tb.astype(np.uint32) << 16).view(np.float32)
            df = (db.astype(np.uint32) << 16).view(np.float32)
            tok, prob = O.topf(tb, db, T, F)
        else:
            tf, df = t, d
            tok, prob = O.topf(t, d, T, F)
        etok, eprob = expected_topf(tf, df, T, F)
        assert (tok == etok).all()
        assert np.allclose(prob, eprob, rtol=1e-12, atol=1e-15)


def check_topf_fallback_and_invalid(O):
    rng = np.random.default_rng(8)
    V, gamma = 40, 2
    t = rng.standard_normal((3, gamma + 1, V)).astype(np.float32)
    d = t[:, :gamma].copy()                  # q = p: the residual vanishes -> p_n
    T = np.array([1.0, -1.0, 1.0], np.float32)  # sequence 1: invalid temperature
    t[2, 1, 5] = np.nan                      # sequence 2: a bad row
    F = [4, 4, 4]
    tok, prob = O.topf(t, d, T, F)
    etok, eprob = expected_topf(t[:1], d[:1], T[:1], F)
    assert (tok[0] == etok[0]).all() and np.allclose(prob[0], eprob[0], rtol=1e-12)
    p0 = _softmax64(t[0, 0], 1.0)
    assert tok[0, 0] == int(np.argmax(p0))   # the fallback is p_0 itself
    assert (tok[1] == -1).all() and (prob[1] == 0).all()
    assert (tok[2] == -1).all() and (prob[2] == 0).all()


def check_topf_properties(O):
    """Definition-level properties on random rows: every listed token outweighs
    every token left out, the list is in decreasing probability, slots past the
    positive tokens are empty, and the probabilities are at most one in total."""
    rng = np.random.default_rng(11)
    V, gamma, B = 30, 3, 5
    t = (rng.standard_normal((B, gamma + 1, V)) * 3).astype(np.float32)
    d = (0.5 * t[:, :gamma] + rng.standard_normal((B, gamma, V))).astype(np.float32)
    T = np.ones(B, np.float32)
    F = [6, 6, 6, 40]                        # the bonus list is longer than V
    tok, prob = O.topf(t, d, T, F)
    off = np.concatenate([[0], np.cumsum(F)])
    for b in range(B):
        for n in range(gamma + 1):
            p = _softmax64(t[b, n], 1.0)
            w = np.maximum(0.0, p - _softmax64(d[b, n], 1.0)) if n < gamma else p
            w = w / w.sum()
            ids = tok[b, off[n]:off[n + 1]]
            pr = prob[b, off[n]:off[n + 1]]
            real = ids[ids >= 0]
            assert np.all(np.diff(pr[: len(real)]) <= 1e-15)
            assert np.all(ids[len(real):] == -1) and np.all(pr[len(real):] == 0)
            left = np.setdiff1d(np.arange(V), real)
            if len(left) and len(real):
                assert w[left].max() <= w[real].min() + 1e-15
            assert pr.sum() <= 1 + 1e-12
            if F[n] >= V:
                assert len(real) == int((w > 0).sum())


def check_cache_lookup(O):
    F = [2, 1, 3]                            # gamma = 2, slots 0-1 | 2 | 3-5
    out_t = np.array([[7, -1, -1], [4, 9, -1], [4, 5, 6], [4, 5, 11], [-1, -1, -1]], np.int32)
    out_n = np.array([0, 1, 2, 2, 0], np.int32)
    cache = np.array([[3, 7, 9, 1, 2, 3],    # n=0, token 7 in slot 1
                      [9, 9, 8, 9, 9, 9],    # n=1, token 9 not in slot 2 (8): miss
                      [0, 0, 0, 5, 6, 6],    # n=2, token 6: first match slot 4
                      [11, 11, 11, 1, 2, 3], # n=2, token 11 only outside its slots: miss
                      [-1, 0, 0, 0, 0, 0]],  # no extra token: miss
                     np.int32)
    assert O.cache_lookup(out_t, out_n, cache, F).tolist() == [1, -1, 4, -1, -1]


def check_outcome_in_its_distribution(O):
    """The extra token verify emits after outcome n has positive probability under
    that outcome's distribution; with a list as long as V it is found in the cache
    built from these lists, in the slot that holds it."""
    rng = np.random.default_rng(21)
    V, gamma, B = 24, 3, 40
    t = (rng.standard_normal((B, gamma + 1, V)) * 2).astype(np.float32)
    d = (t[:, :gamma] + rng.standard_normal((B, gamma, V))).astype(np.float32)
    toks = rng.integers(0, V, (B, gamma)).astype(np.int32)
    T = np.ones(B, np.float32)
    ua = ((rng.integers(0, 2 ** 23, (B, gamma)) * 2 + 1) * 2.0 ** -24).astype(np.float32)
    ur = ((rng.integers(0, 2 ** 23, B) * 2 + 1) * 2.0 ** -24).astype(np.float32)
    r = O.verify(t, d, toks, T, ua, ur)
    F = [V] * (gamma + 1)
    tok, prob = O.topf(t, d, T, F)
    slot = O.cache_lookup(r.out_tokens, r.n_accepted, tok, F)
    for b in range(B):
        n = r.n_accepted[b]
        x = r.out_tokens[b, n]
        assert slot[b] >= 0 and tok[b, slot[b]] == x and prob[b, slot[b]] > 0


ALL_TOPF_CHECKS = [check_fanout_closed_forms, check_topf_hand_case, check_topf_numpy,
                   check_topf_fallback_and_invalid, check_topf_properties, check_cache_lookup,
                   check_outcome_in_its_distribution]
