"""GPU parity of token-tree verification and pruning (SpecLA, Metodologia 1 and
3; Speculative Speculative Decoding, "Significado e Impacto"): spec_verify_tree
and spec_verify_tree_prune, through the C ABI, against the fp64 oracle.

Bar: accepted nodes, tokens, n_accepted and status equal to the oracle's on
every sequence outside the oracle's near-tie band (a test or an inverse-CDF
gap within the band of the fp32 weights; counted, and required to be a small
minority); the normalisers of the rows the walk read within 1e-5 relative and
NaN for the others.  Pruning: cumulative log-probabilities within 1e-6 absolute
plus 1e-9 relative, the keep mask equal where no path sum lies within that of
the threshold."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_84_b200 import binding, workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def run_gpu(w, keep=None):
    d = binding.tree_to_device(w, DEV)
    kp = None if keep is None else torch.from_numpy(np.ascontiguousarray(keep, np.int32)).to(DEV)
    out = binding.tree_verify(d["target"], d["draft"], d["parent"], d["tokens"], d["temperature"], d["u_accept"],
                              d["u_resample"], kp, return_log_norm=True, return_row_status=True)
    return [x.cpu().numpy() for x in out]


def run_oracle(w, keep=None):
    return oracle.tree_verify(w.target, w.draft, w.parent, w.tokens, w.temperature, w.u_accept, w.u_resample,
                              keep, bf16=(w.dtype == "bf16"))


def assert_tree_parity(w, keep=None, max_near_frac=0.15):
    nodes, toks, n, ln, st = run_gpu(w, keep)
    r = run_oracle(w, keep)
    sure = r.near_tie == 0
    assert sure.sum() >= (1 - max_near_frac) * w.B, (w.name, int((~sure).sum()))
    bad = np.nonzero(sure & ((st != r.row_status) | (n != r.n_accepted) | (toks != r.out_tokens).any(1)
                             | (nodes != r.out_nodes).any(1)))[0]
    assert bad.size == 0, (w.name, bad[:8], st[bad[:4]], r.row_status[bad[:4]], toks[bad[:2]], r.out_tokens[bad[:2]])
    for b in np.nonzero(sure)[0]:
        got, want = ln[b], r.log_norm[b]
        assert (np.isnan(got) == np.isnan(want)).all(), (w.name, b, got, want)
        f = ~np.isnan(want)
        assert np.allclose(got[f], want[f], rtol=1e-5, atol=1e-6), (w.name, b)
    return int((~sure).sum())


def test_tree_t3_full():
    """B = 64 trees of shape (3, 2, 1) (16 nodes) over V = 128256, bf16, rho 0.9,
    T = 1: the bench workload, every sequence."""
    w = W.make_tree(64, (3, 2, 1), 128256, "bf16", seed=91, name="t3")
    assert_tree_parity(w)


@pytest.mark.parametrize("B,branching,V,dt,T", [
    (24, (3, 2, 1), 32000, "bf16", [1.0, 0.7, 0.0, 1.7]),
    (9, (8,), 4096, "f32", 1.0),
    (7, (1,) * 12, 1000, "bf16", [0.5, 1.0, 0.0]),
    (5, (2, 2, 2, 2, 2), 333, "f32", 1.0),
    (3, (3, 3, 3), 32003, "bf16", [1.0, 0.0, 0.8]),
    (16, (4, 1), 7, "f32", 1.0),
    (4, (2,), 1, "bf16", 1.0),
    (300, (2, 1), 2048, "bf16", 1.0),
    (1, (5, 2), 151936, "bf16", 1.0),
    (2, (3, 2), 64000, "f32", [1.0, 0.0]),
])
def test_tree_shapes(B, branching, V, dt, T):
    """Ragged and aligned vocabularies (scalar and vector loads), wide, deep and
    bushy trees up to 63 nodes, greedy and mixed temperatures, clusters of 1 to 8
    CTAs per tree (B = 1 .. 300)."""
    w = W.make_tree(B, branching, V, dt, seed=7 + V + B, T=T, rho=0.8)
    assert_tree_parity(w)


def test_tree_chain_matches_spec_verify():
    """A chain through spec_verify_tree gives spec_verify's outputs (both GPU)."""
    for name in ("c2", "c3"):
        wc = W.make_workload(name, B=16)
        d = binding.to_device(wc, DEV)
        t_ref, n_ref = binding.verify(d["target"], d["draft"], d["draft_tokens"], d["temperature"], d["u_accept"],
                                      d["u_resample"])
        B, g1, V = wc.target.shape
        par = torch.arange(-1, g1 - 1, dtype=torch.int32, device=DEV).repeat(B, 1).contiguous()
        tok = torch.cat([torch.zeros((B, 1), dtype=torch.int32, device=DEV), d["draft_tokens"]], 1).contiguous()
        dft = torch.cat([d["draft"], torch.zeros_like(d["target"][:, :1])], 1).contiguous()
        ua = torch.cat([torch.full((B, 1), 0.5, device=DEV), d["u_accept"]], 1).contiguous()
        nodes, toks, n = binding.tree_verify(d["target"], dft, par, tok, d["temperature"], ua, d["u_resample"])
        r = oracle.verify(wc.target, wc.draft, wc.draft_tokens, wc.temperature, wc.u_accept, wc.u_resample)
        sure = r.near_tie == 0
        assert (toks.cpu().numpy()[sure] == t_ref.cpu().numpy()[sure]).all(), name
        assert (n.cpu().numpy()[sure] == n_ref.cpu().numpy()[sure]).all(), name


def test_tree_keep_mask_and_prune():
    """spec_verify_tree_prune against the oracle's pruning, then verification of
    the pruned trees (the keep mask) against the oracle's."""
    for T in (1.0, 0.0, [0.7, 1.0, 0.0, 1.3]):
        w = W.make_tree(12, (3, 2, 2), 8000, "bf16", seed=41, T=T, rho=0.85)
        d = binding.tree_to_device(w, DEV)
        for thr in (-np.inf, -18.0, -9.0, 0.0):
            keep, cum = binding.tree_prune(d["draft"], d["parent"], d["tokens"], d["temperature"], thr)
            keep, cum = keep.cpu().numpy(), cum.cpu().numpy()
            ek, ec = oracle.tree_prune(w.draft, w.parent, w.tokens, w.temperature, thr, bf16=True)
            fin = np.isfinite(ec)
            assert (np.isnan(cum) == np.isnan(ec)).all() and (np.isneginf(cum) == np.isneginf(ec)).all()
            assert np.allclose(cum[fin], ec[fin], rtol=1e-9, atol=1e-6)
            clear = ~(np.abs(np.where(fin, ec, 0.0) - (thr if np.isfinite(thr) else 0.0)) < 1e-5)
            assert (keep[clear] == ek[clear]).all(), (T, thr)
            assert_tree_parity(w, keep=ek)


def test_tree_edge_cases():
    """Bad parent indices (32), bad tokens in nodes that take part (1) and in masked
    ones (nothing), NaN / +inf / all -inf rows that the walk reads (2) and that it
    does not (nothing), bad uniforms (16), bad temperatures (4)."""
    w = W.make_tree(16, (2, 2), 300, "f32", seed=5, T=1.0)
    B, N, V = w.B, w.N, w.V
    par, tok, ua, ur = w.parent.copy(), w.tokens.copy(), w.u_accept.copy(), w.u_resample.copy()
    tgt, dft, T = w.target.copy(), w.draft.copy(), w.temperature.copy()
    keep = np.ones((B, N), np.int32)
    par[0, 3] = 3                 # 32
    par[1, 0] = 0                 # 32
    tok[2, 1] = V                 # 1
    tok[3, 4] = -1; keep[3, 4] = 0  # masked: nothing
    tgt[4, 0, 5] = np.nan         # the root is always read: 2
    tgt[5, 6] = np.inf            # node 6 (a leaf under node 2): read only if the walk goes there
    dft[6, 0] = -np.inf           # the root's draft row: 2
    dft[7, 5] = np.nan            # a leaf's draft row: never read
    ua[8, 2] = 1.0                # 16
    ur[9] = np.nan                # 16
    ua[10, 0] = 7.0               # the root's entry is unused
    T[11] = -1.0                  # 4
    T[12] = 1e-7                  # 4
    T[13] = 0.0; ua[13] = 5.0; ur[13] = -1.0  # greedy reads no uniform
    we = W.TreeWorkload("edges", "f32", tgt, dft, par, tok, T, ua, ur)
    nodes, toks, n, ln, st = run_gpu(we, keep)
    r = run_oracle(we, keep)
    assert (st == r.row_status).all(), (st, r.row_status)
    assert list(st[[0, 1, 2, 4, 6, 8, 9, 11, 12]]) == [32, 32, 1, 2, 2, 16, 16, 4, 4]
    assert st[3] in (0, 8) and st[7] in (0, 8) and st[10] in (0, 8) and st[13] == 0
    sure = r.near_tie == 0
    assert (toks[sure] == r.out_tokens[sure]).all() and (n[sure] == r.n_accepted[sure]).all()


def test_tree_prune_edge_cases():
    """Pruning on malformed sequences: a bad parent index, a node after its own
    index, a bad or NaN temperature (every node kept, cum NaN); a token outside
    [0, V) and a NaN draft row on a kept path (NaN entries, nodes kept); greedy and
    ragged rows (scalar loads); every output equal to the oracle's."""
    for V, dt in ((300, "f32"), (333, "bf16"), (4096, "bf16")):
        w = W.make_tree(10, (2, 2), V, dt, seed=17 + V, T=[1.0, 0.7, 0.0, 1.3, 1.0, 1.0, 0.0, 1.0, 1.0, 2.0])
        par, tok, dft, T = w.parent.copy(), w.tokens.copy(), w.draft.copy(), w.temperature.copy()
        par[0, 3] = 3                 # a node its own parent
        par[1, 0] = 0                 # the root with a parent
        T[4] = -1.0                   # bad temperature
        T[5] = np.nan
        tok[7, 2] = V                 # a token outside the vocabulary
        dft[8, 1] = np.nan if dt == "f32" else 0x7fc0  # a NaN row with children
        we = W.TreeWorkload("prune_edges", dt, w.target, dft, par, tok, T, w.u_accept, w.u_resample)
        d = binding.tree_to_device(we, DEV)
        for thr in (-np.inf, -9.0):
            keep, cum = binding.tree_prune(d["draft"], d["parent"], d["tokens"], d["temperature"], thr)
            keep, cum = keep.cpu().numpy(), cum.cpu().numpy()
            ek, ec = oracle.tree_prune(dft, par, tok, T, thr, bf16=(dt == "bf16"))
            assert (np.isnan(cum) == np.isnan(ec)).all(), (V, thr)
            fin = np.isfinite(ec)
            assert (np.isneginf(cum) == np.isneginf(ec)).all()
            assert np.allclose(cum[fin], ec[fin], rtol=1e-9, atol=1e-6), (V, thr)
            clear = ~(np.abs(np.where(fin, ec, 0.0) - (thr if np.isfinite(thr) else 0.0)) < 1e-5)
            assert (keep[clear] == ek[clear]).all(), (V, thr)
            for b in (0, 1, 4, 5):
                assert (keep[b] == 1).all() and np.isnan(cum[b]).all(), (V, b)
