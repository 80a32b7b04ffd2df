"""GPU parity of the speculation cache's side of an outcome: spec_verify_topf
(the F_n most probable tokens of the extra token's distribution per outcome n)
and spec_verify_cache_lookup, through the C ABI, against the fp64 oracle.

The ranking is compared where it is unique: the k-th largest probability must
match the oracle's k-th largest (1e-5 relative, plus the fp32 rounding of the
difference p - q below), every listed token's oracle probability must match that
rank's, and where the oracle's k-th and (k+1)-th probabilities are further apart
than that tolerance the tokens must be the same; tokens of equal probability (a
near tie) may come in either order.
The lookup is integer work: bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import parity
from speculative_decoding_verification_84_b200 import binding, workloads as W

pytestmark = pytest.mark.gpu

# fp32 weights: p and q each carry a relative error of at most about 1e-6 (the
# exp2 unit's 2 ulp plus the rounding of its argument), so a residual weight
# p - q carries an absolute error of about 1e-6 (p + q); SCALE_TOL bounds that
# with margin, in units of (p + q) / S.
RTOL, ATOL, SCALE_TOL = 1e-5, 1e-7, 4e-6


def _widen(a, dt):
    if dt == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32)
    return a


def _distributions(w, b, n):
    """The oracle's (numpy) distribution of the extra token after outcome n, and
    the scale of its fp32 rounding per token: (p + q) / S for the residual (the
    difference of two rounded terms), p / S otherwise."""
    gamma = w.gamma
    t = _widen(w.target, w.dtype)[b].astype(np.float64)
    d = _widen(w.draft, w.dtype)[b].astype(np.float64)
    T = float(w.temperature[b])

    def sm(row):
        z = row / T
        z = z - z.max()
        e = np.exp(z)
        return e / e.sum()
    p = sm(t[n])
    if n < gamma:
        q = sm(d[n])
        r = np.maximum(0.0, p - q)
        if not r.sum() >= oracle.RESIDUAL_MIN:
            return p, p
        return r / r.sum(), (p + q) / r.sum()
    return p, p


def _check_topf(w, F, tok, prob):
    etok, eprob = oracle.topf_workload(w, F)
    off = np.concatenate([[0], np.cumsum(F)])
    same = swapped = 0
    for b in range(w.B):
        for n in range(w.gamma + 1):
            g_t, g_p = tok[b, off[n]:off[n + 1]], prob[b, off[n]:off[n + 1]]
            o_t, o_p = etok[b, off[n]:off[n + 1]], eprob[b, off[n]:off[n + 1]]
            if w.temperature[b] == 0 or (o_t < 0).all():
                assert (g_t == o_t).all() and np.allclose(g_p, o_p, rtol=RTOL, atol=ATOL), (b, n)
                continue
            dist, scale = _distributions(w, b, n)

            def tol(v, pr):
                return RTOL * pr + SCALE_TOL * scale[v] + ATOL
            for s in range(len(o_t)):
                if o_t[s] < 0 or o_p[s] < ATOL:
                    # empty slot, or weight too small for fp32 to rank: the GPU slot
                    # is empty or holds a token of (near) zero probability
                    assert g_t[s] < 0 or dist[g_t[s]] < 10 * ATOL + SCALE_TOL * scale[g_t[s]], (b, n, s)
                    continue
                assert g_t[s] >= 0, (b, n, s)
                t_o = tol(o_t[s], o_p[s])
                assert abs(dist[g_t[s]] - o_p[s]) <= t_o + tol(g_t[s], dist[g_t[s]]), (b, n, s, g_t[s], o_t[s])
                assert abs(g_p[s] - o_p[s]) <= t_o + tol(g_t[s], dist[g_t[s]]), (b, n, s, g_p[s], o_p[s])
                nxt = o_p[s + 1] if s + 1 < len(o_p) else 0.0
                prv = o_p[s - 1] if s > 0 else np.inf
                t_n = tol(o_t[s + 1], nxt) if s + 1 < len(o_p) and o_t[s + 1] >= 0 else ATOL
                t_p = tol(o_t[s - 1], prv) if s > 0 else 0.0
                unique = (o_p[s] - nxt > t_o + t_n) and (prv - o_p[s] > t_o + t_p)
                if g_t[s] == o_t[s]:
                    same += 1
                else:
                    assert not unique, (b, n, s, g_t[s], o_t[s])
                    swapped += 1
    return same, swapped


def _run(w, F):
    d = binding.to_device(w)
    toks, n, ln, st = binding.verify(**d, return_log_norm=True, return_row_status=True)
    tok, prob = binding.topf(d["target"], d["draft"], d["temperature"], ln, st, F)
    slot = binding.cache_lookup(toks, n, tok, F)
    torch.cuda.synchronize()
    return toks.cpu().numpy(), n.cpu().numpy(), tok.cpu().numpy(), prob.cpu().numpy(), slot.cpu().numpy()


CASES = [
    ("c1", None), ("c2", None), ("c3", range(12)), ("c5", range(600)),
]


@pytest.mark.parametrize("name,seqs", CASES)
def test_topf_configs(name, seqs):
    w = W.make_workload(name, **({} if seqs is None else ({"B": len(seqs)} if name == "c5" else {"seqs": seqs})))
    F = np.minimum(binding.fanout(0.7, w.gamma, 8 * (w.gamma + 1)), binding.MAX_TOPF)
    gt, gn, tok, prob, slot = _run(w, F)
    same, swapped = _check_topf(w, F, tok, prob)
    print(f"{name}: {same} slots identical, {swapped} near-tie swaps")
    # the lookup, with the GPU's own lists as the cache: bit-exact against the oracle's rule
    assert (slot == oracle.cache_lookup(gt, gn, tok, F)).all()


@pytest.mark.parametrize("B,gamma,V,dt", [(9, 3, 1000, "f32"), (5, 4, 4097, "bf16"), (7, 2, 33, "f32"),
                                          (3, 6, 32000, "bf16"), (4, 1, 257, "bf16")])
def test_topf_ragged_and_greedy(B, gamma, V, dt):
    """Odd V (scalar loads), greedy and invalid sequences, lists longer than the
    tokens of positive probability, an outcome with no slots."""
    T = np.resize(np.array([1.0, 0.0, 0.7, -1.0, 1.5], np.float32), B)
    w = W.make_random(B, gamma, V, dt, seed=300 + V + B, T=T)
    F = np.resize(np.array([32, 0, 5, 1, 17, 3, 2], np.int32), gamma + 1)
    gt, gn, tok, prob, slot = _run(w, F)
    _check_topf(w, F, tok, prob)
    assert (slot == oracle.cache_lookup(gt, gn, tok, F)).all()
    et, _ = oracle.topf_workload(w, F)
    assert (oracle.cache_lookup(gt, gn, et, F) >= -1).all()


def test_topf_vanished_residual_and_bad_rows():
    import oracle_pins
    rng = np.random.default_rng(4)
    V, gamma = 256, 2
    vanished = oracle_pins.vanished_residual_cases(V)
    B = 4 + len(vanished)
    tgt = (rng.standard_normal((B, gamma + 1, V)) * 2).astype(np.float32)
    dft = (tgt[:, :gamma] + rng.standard_normal((B, gamma, V))).astype(np.float32)
    tgt[1, 2, 7] = np.nan        # a bad row: no lists
    dft[2, 0, :] = -np.inf       # an all -inf draft row: bad
    for i, (lt, ld, x, u) in enumerate(vanished):
        tgt[4 + i, 0], dft[4 + i, 0] = lt, ld
    toks = rng.integers(0, V, (B, gamma)).astype(np.int32)
    ua, ur = W.draw_uniforms(rng, (B, gamma)), W.draw_uniforms(rng, (B,))
    w = W.Workload("topf-edges", "f32", tgt, dft, toks, np.ones(B, np.float32), ua, ur)
    F = np.array([8, 8, 8], np.int32)
    gt, gn, tok, prob, slot = _run(w, F)
    _check_topf(w, F, tok, prob)
    assert (tok[1] == -1).all() and (tok[2] == -1).all()
    assert (slot == oracle.cache_lookup(gt, gn, tok, F)).all()


def test_outcome_found_in_full_cache():
    """With lists as long as V the emitted extra token is always in the cache (it
    has positive probability), except after near-tie draws."""
    w = W.make_random(40, 3, 24, "f32", seed=21, T=np.ones(40, np.float32))
    F = np.full(4, 24, np.int32)
    gt, gn, tok, prob, slot = _run(w, F)
    ref = oracle.verify_workload(w)
    near = (ref.accept_gap < parity.BAND) | (ref.cdf_gap < parity.BAND)
    assert ((slot >= 0) | near).all()
