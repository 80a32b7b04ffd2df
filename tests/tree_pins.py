"""Pins of the oracle's tree verification and pruning (SpecLA, Metodologia 1,
"Kernels de Verificacao de Topologia Conscientes"; Metodologia 3, "Poda Guiada
por Confianca"; Speculative Speculative Decoding, "Significado e Impacto": token
trees), each against something other than the tree code itself:

* a chain is the chain verifier's case: the tree oracle on chains must give
  sv_oracle_verify's results (itself pinned), and pass the chain pins that do
  not depend on rows past the walk;
* hand-worked three-token cases of the multi-candidate rule;
* numpy first-argmax for greedy trees;
* the output law: over many independent trees whose siblings are drawn from q,
  the first emitted token follows the target's p at the root, and after an
  accepted draft x the second follows the target's p at context x (chi-square);
* the rows a walk reads, the node mask and the status bits;
* pruning: cumulative log-probabilities against numpy log-softmax sums along the
  paths, and the keep rule.

Every check takes an object ``O`` with ``tree_verify``, ``tree_prune`` and
``verify`` (the oracle module, or a stand-in built from a copy of the oracle
with a planted mistake)."""
from __future__ import annotations

import math

import numpy as np

import oracle_pins as CP


# ----------------------------------------------------------------- helpers

def chain_to_tree(target, draft, tokens, ua):
    """Chain inputs of sv_oracle_verify ([B][g+1][V], [B][g][V], [B][g], [B][g]) as
    a tree: node i's parent is i - 1, the leaf's draft row is never read."""
    target = np.ascontiguousarray(target)
    B, N, V = target.shape
    par = np.tile(np.arange(-1, N - 1, dtype=np.int32), (B, 1))
    tok = np.concatenate([np.zeros((B, 1), np.int32), np.asarray(tokens, np.int32)], axis=1)
    dft = np.concatenate([np.asarray(draft), np.zeros((B, 1, V), draft.dtype)], axis=1)
    u = np.concatenate([np.full((B, 1), 0.5, np.float32), np.asarray(ua, np.float32)], axis=1)
    return target, dft, par, tok, u


class ChainResult:
    def __init__(self, r, gamma):
        N = gamma + 1
        self.out_tokens = r.out_tokens
        self.n_accepted = r.n_accepted
        self.log_norm = np.concatenate([r.log_norm[:, :N], r.log_norm[:, N:N + gamma]], axis=1)
        self.row_status = r.row_status
        self.near_tie = r.near_tie
        self.accept_gap = r.accept_gap
        self.cdf_gap = r.cdf_gap


def chain_adapter(O):
    """A ``verify`` callable that runs the tree oracle on chains."""
    def verify(target, draft, tokens, temperature, ua, ur, *, bf16=None, n_threads=0, lib=None):
        t, d, par, tok, u = chain_to_tree(target, draft, tokens, ua)
        r = O.tree_verify(t, d, par, tok, temperature, u, ur, bf16=bf16)
        return ChainResult(r, np.asarray(target).shape[1] - 1)
    return verify


def _logits(p):
    """float32 logits whose softmax is p to float32 precision."""
    return np.log(np.asarray(p, np.float64)).astype(np.float32)


def _one(O, tgt_rows, dft_rows, par, tok, ua, ur, T=1.0, keep=None):
    tgt = np.asarray(tgt_rows, np.float32)[None]
    dft = np.asarray(dft_rows, np.float32)[None]
    r = O.tree_verify(tgt, dft, np.asarray(par, np.int32)[None], np.asarray(tok, np.int32)[None],
                      np.asarray([T], np.float32), np.asarray(ua, np.float32)[None], np.asarray([ur], np.float32),
                      None if keep is None else np.asarray(keep, np.int32)[None])
    return r


# ----------------------------------------------------------------- chains

def check_chain_equals_verify(O):
    """Random chains (f32 and bf16, T in {0, 0.7, 1, 1.7}, ragged V, gamma 1-6): every
    output of the tree oracle equals sv_oracle_verify's; its normalisers are those
    of the rows the walk read (the others NaN)."""
    from speculative_decoding_verification_84_b200 import workloads as W
    cases = [(6, 1, 7, "f32", 1.0), (8, 4, 50, "f32", [0.0, 0.7, 1.0, 1.7] * 2), (5, 6, 129, "bf16", 0.7),
             (4, 3, 1000, "bf16", [1.0, 0.0, 1.7, 1.0]), (3, 2, 1, "f32", 1.0)]
    for B, g, V, dt, T in cases:
        w = W.make_random(B, g, V, dt, seed=17 + V, T=T, draft_noise=0.8)
        c = O.verify(w.target, w.draft, w.draft_tokens, w.temperature, w.u_accept, w.u_resample)
        t, d, par, tok, u = chain_to_tree(w.target, w.draft, w.draft_tokens, w.u_accept)
        r = O.tree_verify(t, d, par, tok, w.temperature, u, w.u_resample)
        assert (r.out_tokens == c.out_tokens).all(), (B, g, V)
        assert (r.n_accepted == c.n_accepted).all()
        assert (r.row_status == c.row_status).all()
        assert (r.near_tie == c.near_tie).all()
        assert (r.accept_gap == c.accept_gap).all() and (r.cdf_gap == c.cdf_gap).all()
        N = g + 1
        for b in range(B):
            n = int(c.n_accepted[b])
            read_t = list(range(n + 1))
            read_d = [j for j in range(min(n + 1, g))] if w.temperature[b] > 0 else []
            if w.temperature[b] == 0:
                assert np.isnan(r.log_norm[b]).all()
                continue
            for j in range(N):
                if j in read_t:
                    assert r.log_norm[b, j] == c.log_norm[b, j]
                else:
                    assert np.isnan(r.log_norm[b, j])
            for j in range(N):
                if j in read_d:
                    assert r.log_norm[b, N + j] == c.log_norm[b, N + j]
                else:
                    assert np.isnan(r.log_norm[b, N + j])


CHAIN_PINS = [CP.check_greedy_argmax, CP.check_accept_boundary, CP.check_inverse_cdf_searchsorted,
              CP.check_residual_vanished, CP.check_oracle_partition]


def check_chain_pins_through_tree(O):
    """The chain pins whose inputs keep every row valid, run on the tree oracle."""
    v = chain_adapter(O)
    for check in CHAIN_PINS:
        check(v)


# ----------------------------------------------------------------- the multi-candidate rule by hand

P3 = [0.5, 0.3, 0.2]
Q3 = [0.2, 0.5, 0.3]


def check_siblings_by_hand(O):
    """Root with two children, V = 3, p = (0.5, 0.3, 0.2), q = (0.2, 0.5, 0.3).
    (a) tokens (1, 1), u = 0.7: 0.7 > p1/q1 = 0.6 rejects; P becomes
        norm(max(0, p - q)) = (1, 0, 0); the second child has P(1) = 0 and is
        rejected; the extra token comes from max(0, P - q) = (0.8, 0, 0): token 0.
    (b) tokens (1, 1), u = 0.59 < 0.6: the first child is accepted (n = 1) and the
        walk moves to node 1, a leaf: bonus token from node 1's target row.
    (c) tokens (1, 0), u1 = 0.7: rejected as in (a); then P(0)/q(0) = 1/0.2 = 5, so
        the second child is accepted for any u (u2 = 0.999).
    (d) tokens (2, 1), u1 = 0.9 > p2/q2 = 0.667 rejects; P = (1, 0, 0); the second
        child (token 1) is rejected; extra token 0.
    (e) the children are tried in index order: tokens (0, 1), u = (0.999, ...):
        p0/q0 = 2.5 accepts node 1 first."""
    lt, ld = _logits(P3), _logits(Q3)
    leaf_t = _logits([0.1, 0.1, 0.8])  # the children's own rows: a bonus from here is token 2 for u = 0.5
    tg = [lt, leaf_t, leaf_t]
    dg = [ld, ld, ld]
    par = [-1, 0, 0]
    r = _one(O, tg, dg, par, [0, 1, 1], [0.5, 0.7, 0.5], 0.5)
    assert r.n_accepted[0] == 0 and list(r.out_tokens[0]) == [0, -1, -1] and r.row_status[0] == 0
    r = _one(O, tg, dg, par, [0, 1, 1], [0.5, 0.59, 0.5], 0.5)
    assert r.n_accepted[0] == 1 and list(r.out_nodes[0]) == [1, -1, -1] and list(r.out_tokens[0]) == [1, 2, -1]
    r = _one(O, tg, dg, par, [0, 1, 0], [0.5, 0.7, 0.999], 0.5)
    assert r.n_accepted[0] == 1 and list(r.out_nodes[0]) == [2, -1, -1] and list(r.out_tokens[0]) == [0, 2, -1]
    r = _one(O, tg, dg, par, [0, 2, 1], [0.5, 0.9, 0.01], 0.99)
    assert r.n_accepted[0] == 0 and list(r.out_tokens[0]) == [0, -1, -1]
    r = _one(O, tg, dg, par, [0, 0, 1], [0.5, 0.999, 0.01], 0.5)
    assert r.n_accepted[0] == 1 and list(r.out_nodes[0]) == [1, -1, -1]


def check_second_sibling_boundary(O):
    """After one rejection the second child is tested against the residual: with
    p = (0.5, 0.3, 0.2), q = (0.3, 0.2, 0.5), the first child (token 2: 0.4) is
    rejected by u = 0.5, P = norm(max(0, p - q)) = (0.2, 0.1, 0) / 0.3, and the
    second child (token 0) has P0/q0 = (2/3)/0.3 = 20/9 > 1: accepted; with token 1,
    P1/q1 = (1/3)/0.2 = 5/3: accepted; u just below / above such a ratio below 1
    is checked on p = (0.4, 0.35, 0.25), q = (0.1, 0.3, 0.6): after rejecting token 2
    (ratio 0.417, u = 0.5) P = (0.3, 0.05, 0)/0.35, token 1's ratio is
    (0.05/0.35)/0.3 = 0.47619: u = 0.4761 accepts, 0.4763 rejects."""
    for p, q, tok2, u2, acc in [([0.5, 0.3, 0.2], [0.3, 0.2, 0.5], 0, 0.999, True),
                                ([0.5, 0.3, 0.2], [0.3, 0.2, 0.5], 1, 0.999, True),
                                ([0.4, 0.35, 0.25], [0.1, 0.3, 0.6], 1, 0.4761, True),
                                ([0.4, 0.35, 0.25], [0.1, 0.3, 0.6], 1, 0.4763, False)]:
        lt, ld = _logits(p), _logits(q)
        r = _one(O, [lt, lt, lt], [ld, ld, ld], [-1, 0, 0], [0, 2, tok2], [0.5, 0.5, u2], 0.3)
        assert (r.n_accepted[0] == 1) == acc, (p, q, tok2, u2)
        if acc:
            assert r.out_nodes[0, 0] == 2


def check_greedy_tree(O):
    """T = 0: the first child whose token is numpy.argmax of the node's target row
    (first index on ties) is accepted; the walk descends; the extra token is the
    argmax of the last node's row."""
    rng = np.random.default_rng(5)
    V = 6
    for trial in range(40):
        # root with 3 children, the first two children with 2 children each
        par = [-1, 0, 0, 0, 1, 1, 2, 2]
        N = len(par)
        tg = (rng.integers(0, 3, size=(N, V))).astype(np.float32)  # small integers: ties
        tok = [0] + list(rng.integers(0, V, size=N - 1))
        r = _one(O, tg, np.zeros((N, V), np.float32), par, tok, [0.5] * N, 0.5, T=0.0)
        c, path = 0, []
        while True:
            a = int(np.argmax(tg[c]))
            nxt = next((i for i in range(c + 1, N) if par[i] == c and tok[i] == a), None)
            if nxt is None:
                break
            path.append(nxt)
            c = nxt
        assert r.n_accepted[0] == len(path)
        assert list(r.out_nodes[0, :len(path)]) == path
        assert list(r.out_tokens[0, :len(path) + 1]) == [tok[i] for i in path] + [a]
        assert r.row_status[0] == 0 and np.isnan(r.log_norm[0]).all()


# ----------------------------------------------------------------- the output law

def _chi2_ok(counts, p, alpha=1e-3):
    return CP._chi2_pvalue(np.asarray(counts), np.asarray(p)) > alpha


def check_tree_law(O):
    """Trees whose siblings are drawn independently from q (V = 4; the root has 3
    children, each with 2 children; every node's rows are those of its context, so
    equal tokens give equal rows).  Over 30,000 trees the first emitted token
    follows p at the root and, after an accepted draft x, the second follows p at
    context x (chi-square, p-value > 1e-3 each)."""
    V, T = 4, 1.0
    rng = np.random.default_rng(12)
    # contexts: () -> 0, (x,) -> 1 + x, (x, y) -> 5 + 4x + y
    n_ctx = 1 + V + V * V
    P = rng.dirichlet(np.full(V, 1.5), size=n_ctx)
    Q = rng.dirichlet(np.full(V, 1.5), size=n_ctx)
    LT, LD = _logits(P), _logits(Q)
    par = [-1, 0, 0, 0, 1, 1, 2, 2, 3, 3]
    N = len(par)
    B = 30_000

    def draw(ctx):  # one token per tree from q at each tree's context id
        cdf = np.cumsum(Q[ctx], axis=1)
        return np.minimum((rng.random(ctx.size)[:, None] > cdf).sum(axis=1), V - 1).astype(np.int32)

    ctx = np.zeros((B, N), np.int64)
    tok = np.zeros((B, N), np.int32)
    for i in range(1, N):
        tok[:, i] = draw(ctx[:, par[i]])
        ctx[:, i] = 1 + tok[:, i] if par[i] == 0 else 5 + V * tok[:, par[i]] + tok[:, i]
    tgt = LT[ctx]
    dft = LD[ctx]
    ua = rng.random((B, N)).astype(np.float32)
    ur = rng.random(B).astype(np.float32)
    r = O.tree_verify(tgt, dft, np.tile(np.asarray(par, np.int32), (B, 1)), tok, np.full(B, T, np.float32), ua, ur)
    assert (r.row_status == 0).all()
    p_root = np.exp(tgt[0, 0].astype(np.float64))
    p_root /= p_root.sum()
    first = r.out_tokens[:, 0]
    assert _chi2_ok(np.bincount(first, minlength=V), p_root), np.bincount(first, minlength=V) / B
    for x in range(V):
        sel = (r.n_accepted >= 1) & (first == x)
        if sel.sum() < 2000:
            continue
        px = np.exp(LT[1 + x].astype(np.float64))
        px /= px.sum()
        assert _chi2_ok(np.bincount(r.out_tokens[sel, 1], minlength=V), px), x


# ----------------------------------------------------------------- rows read, masks, status

def check_rows_read_and_status(O):
    """Status 2 only for a bad row the walk reads; 32 for a parent index out of
    range; 1 and 16 only for nodes that take part; a masked child is skipped."""
    V = 8
    rng = np.random.default_rng(3)
    base = rng.standard_normal((4, V)).astype(np.float32)
    par = [-1, 0, 0, 1]
    tg = base.copy()
    dg = base.copy()
    # child 1 (token 0) is rejected for sure: draft puts far more mass on it
    tg[0, 0] = -20.0
    dg[0, 0] = 5.0
    tok = [0, 0, 3, 2]
    u = [0.5, 0.5, 0.0, 0.5]  # u = 0 accepts any token of positive probability
    r = _one(O, tg, dg, par, tok, u, 0.5)
    assert r.row_status[0] == 0 and list(r.out_nodes[0, :1]) == [2] and r.n_accepted[0] == 1
    bad = tg.copy(); bad[1, 2] = np.nan          # node 1 is never visited
    assert _one(O, bad, dg, par, tok, u, 0.5).row_status[0] == 0
    bad = tg.copy(); bad[2, 2] = np.inf          # node 2 is visited
    r = _one(O, bad, dg, par, tok, u, 0.5)
    assert r.row_status[0] == 2 and r.n_accepted[0] == 0 and (r.out_tokens[0] == -1).all()
    bad = dg.copy(); bad[2, :] = -np.inf         # node 2 has no children: its draft row is not read
    assert _one(O, tg, bad, par, tok, u, 0.5).row_status[0] == 0
    bad = dg.copy(); bad[0, :] = -np.inf         # the root's draft row is read
    assert _one(O, tg, bad, par, tok, u, 0.5).row_status[0] == 2
    assert _one(O, tg, dg, [-1, 0, 2, 1], tok, u, 0.5).row_status[0] == 32
    assert _one(O, tg, dg, [0, 0, 0, 1], tok, u, 0.5).row_status[0] == 32
    assert _one(O, tg, dg, par, [0, 0, V, 2], u, 0.5).row_status[0] == 1
    assert _one(O, tg, dg, par, [0, 0, 3, 2], [0.5, 1.0, 0.0, 0.5], 0.5).row_status[0] == 16
    # masking node 1 removes it and its child: node 2 is then the first child, and the
    # bad token and uniform of node 3 (node 1's child) are not looked at
    keep = [1, 0, 1, 1]
    r = _one(O, tg, dg, par, [0, 0, 3, V + 5], [0.5, 7.0, 0.0, 9.0], 0.5, keep=keep)
    assert r.row_status[0] == 0 and list(r.out_nodes[0, :1]) == [2]
    # a masked first child changes which uniform decides: node 2 alone, u = 0.999
    r2 = _one(O, tg, dg, par, tok, [0.5, 0.5, 0.999, 0.5], 0.5, keep=[1, 0, 1, 1])
    p = np.exp(tg[0].astype(np.float64)); p /= p.sum()
    q = np.exp(dg[0].astype(np.float64)); q /= q.sum()
    assert (r2.n_accepted[0] == 1) == (0.999 < p[3] / q[3])


def check_residual_vanished_between_siblings(O):
    """A rejection whose residual mass is 0 (rows equal except at the draft token,
    whose logits sit ~100 below the rest) leaves P = p: status bit 8, and the second
    child is tested against p itself."""
    V = 40
    cases = CP.vanished_residual_cases(V)
    lt, ld, x, _ = cases[0]
    rng = np.random.default_rng(9)
    for y in rng.integers(0, V, size=6):
        y = int(y)
        if y == x:
            continue
        p = CP.fsum_softmax(lt.astype(np.float64), 1.0)
        q = CP.fsum_softmax(ld.astype(np.float64), 1.0)
        for u2 in (0.3, 0.95):
            r = _one(O, [lt, lt, lt], [ld, ld, ld], [-1, 0, 0], [0, x, y], [0.5, 0.75, u2], 0.4)
            assert r.row_status[0] & 8
            want = math.log(u2) < math.log(p[y]) - math.log(q[y])
            if abs(math.log(u2) - (math.log(p[y]) - math.log(q[y]))) > 1e-6:
                assert (r.n_accepted[0] == 1) == want, (y, u2)


# ----------------------------------------------------------------- pruning

def _numpy_logsoftmax(row, T):
    z = row.astype(np.float64) / T
    m = z.max()
    return z - (m + np.log(np.exp(z - m).sum()))


def check_prune_cumulative(O):
    """cum[i] = cum[parent] + log q_parent(tok[i]) (numpy log-softmax, fp64) along
    every path; keep[i] = keep[parent] and cum[i] >= threshold; threshold -inf keeps
    every node, +inf keeps only the root; greedy drafts give 0 or -inf."""
    from speculative_decoding_verification_84_b200 import workloads as W
    rng = np.random.default_rng(4)
    B, V = 6, 300
    par = np.array([-1, 0, 0, 0, 1, 1, 2, 4, 4, 7], np.int32)
    N = par.size
    dft = (rng.standard_normal((B, N, V)) * 2.0).astype(np.float32)
    tok = rng.integers(0, V, size=(B, N)).astype(np.int32)
    T = np.array([1.0, 0.7, 1.3, 1.0, 0.0, 1.0], np.float32)
    for b in range(B):  # greedy sequence: make some children the argmax
        if T[b] == 0:
            for i in (1, 4, 7):
                tok[b, i] = int(np.argmax(dft[b, par[i]]))
    P = np.tile(par, (B, 1))
    for thr in (-np.inf, -12.0, -6.0, np.inf):
        keep, cum = O.tree_prune(dft, P, tok, T, thr)
        for b in range(B):
            want = np.zeros(N)
            for i in range(1, N):
                c = par[i]
                if T[b] == 0:
                    lq = 0.0 if tok[b, i] == int(np.argmax(dft[b, c])) else -np.inf
                else:
                    lq = _numpy_logsoftmax(dft[b, c], T[b])[tok[b, i]]
                want[i] = want[c] + lq
            assert np.allclose(cum[b][np.isfinite(want)], want[np.isfinite(want)], rtol=1e-12, atol=1e-12)
            assert (np.isneginf(cum[b]) == np.isneginf(want)).all()
            k = [1] + [0] * (N - 1)
            for i in range(1, N):
                k[i] = int(k[par[i]] and not (want[i] < thr))
            assert list(keep[b]) == k, (b, thr, list(keep[b]), k)
        if thr == -np.inf:
            assert (keep == 1).all()
        if thr == np.inf:
            assert (keep[:, 1:] == 0).all() and (keep[:, 0] == 1).all()
    # bad inputs are kept (cum NaN), so the verification reports them
    T2 = np.array([np.nan, 1.0, 1.0, 1.0, 1.0, 1.0], np.float32)
    tok2 = tok.copy(); tok2[1, 3] = V
    P2 = P.copy(); P2[2, 5] = 7
    keep, cum = O.tree_prune(dft, P2, tok2, T2, 0.0)
    assert (keep[0] == 1).all() and np.isnan(cum[0]).all()
    assert keep[1, 3] == 1 and np.isnan(cum[1, 3])
    assert (keep[2] == 1).all() and np.isnan(cum[2]).all()


ALL_TREE_CHECKS = [check_chain_equals_verify, check_siblings_by_hand, check_second_sibling_boundary,
                   check_greedy_tree, check_rows_read_and_status, check_residual_vanished_between_siblings,
                   check_tree_law, check_prune_cumulative, check_chain_pins_through_tree]
