"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Bar: n_accepted / out_tokens bit-exact except sequences within 1e-6 of a
decision boundary (counted); per-row log-normaliser within 1e-5 relative;
row status exact.  See parity.py."""
import numpy as np
import pytest
import torch

import oracle
import parity
from speculative_decoding_verification_84_b200 import binding, workloads as W

pytestmark = pytest.mark.gpu


def _report(name, stats):
    print(f"[parity] {name}: {stats}")


@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c5"])
def test_config_full(name):
    """Whole configuration, every sequence compared."""
    w = W.make_workload(name)
    g = parity.run_gpu(w)
    st = parity.compare(g, oracle.verify_workload(w))
    _report(name, st)
    parity.assert_parity(st)


def test_config_c4_full():
    """c4 at full size (B=256, gamma=8, V=151936, greedy / 0.6 / 1.0 by sequence):
    every sequence compared with the oracle."""
    w = W.make_workload("c4")
    g = parity.run_gpu(w)
    st = parity.compare(g, oracle.verify_workload(w))
    _report("c4", st)
    assert st["B"] == 256
    parity.assert_parity(st)


RAGGED = [
    (1, 1, 1, "f32"), (3, 2, 7, "bf16"), (5, 3, 9, "f32"), (2, 7, 1000, "bf16"), (4, 1, 1025, "f32"),
    (3, 4, 4097, "bf16"), (17, 5, 3001, "bf16"), (2, 32, 333, "f32"), (6, 3, 33333, "bf16"),
    (1, 4, 32003, "f32"), (9, 2, 8195, "f32"), (40, 2, 257, "bf16"),
    # rows of at most 256 elements: the short-row kernel with groups of 8, 16 and 32
    # lanes, mixed greedy / sampled groups in one warp, a part-filled last warp
    (37, 4, 64, "f32"), (6, 12, 100, "bf16"), (4, 20, 256, "f32"), (11, 8, 33, "bf16"),
]

# 16-byte-aligned rows of at least 4 KB: the streaming kernels.  Short rows (one
# pass-1 span covers several), gamma = 32 (65 rows per sequence), a ragged last
# tile, draws over more than one block of tile sums, rows whose tile sums do not
# fit in shared memory (more than 4096 tiles), and more sequences than resident
# pass-2 clusters (each cluster finishes and draws several in turn).
ALIGNED = [
    (5, 3, 2056, "bf16"), (2, 32, 1032, "f32"), (7, 4, 40008, "bf16"), (11, 6, 12344, "f32"),
    (1, 2, 250000, "f32"), (3, 1, 600000, "f32"), (90, 2, 4096, "bf16"), (400, 1, 2048, "bf16"),
]


@pytest.mark.parametrize("B,gamma,V,dt", RAGGED)
def test_ragged_shapes(B, gamma, V, dt):
    """Odd vocabulary sizes (misaligned rows, ragged tails), gamma 1..32, mixed T incl. greedy."""
    T = np.array([0.0, 0.4, 1.0, 1.7, 1e-3][: 5] * ((B + 4) // 5), np.float32)[:B]
    w = W.make_random(B, gamma, V, dt, seed=1000 + V + 7 * B + gamma, T=T)
    st = parity.compare(parity.run_gpu(w), oracle.verify_workload(w))
    _report(f"{B}x{gamma}x{V}-{dt}", st)
    parity.assert_parity(st)


@pytest.mark.parametrize("B,gamma,V,dt", ALIGNED)
def test_aligned_shapes(B, gamma, V, dt):
    """Shapes that take the streaming kernels, mixed T incl. greedy."""
    assert (V * (2 if dt == "bf16" else 4)) % 16 == 0
    T = np.array([0.0, 0.4, 1.0, 1.7, 1e-3][: 5] * ((B + 4) // 5), np.float32)[:B]
    w = W.make_random(B, gamma, V, dt, seed=2000 + V + 7 * B + gamma, T=T)
    st = parity.compare(parity.run_gpu(w), oracle.verify_workload(w))
    _report(f"{B}x{gamma}x{V}-{dt}", st)
    parity.assert_parity(st)


@pytest.mark.parametrize("V", [64, 300, 4096])
def test_edge_cases(V):
    """NaN / +inf / all -inf rows, out-of-range tokens, invalid temperatures, masked vocab,
    uniforms outside [0, 1), and residuals that vanish after a rejection
    (V = 64: the short-row kernel; V = 300: the general kernels; V = 4096 f32, 16 KB
    rows: the streaming kernels)."""
    import oracle_pins
    rng = np.random.default_rng(9)
    vanished = oracle_pins.vanished_residual_cases(V)
    B, gamma = 20 + len(vanished), 3
    tgt = (rng.standard_normal((B, gamma + 1, V)) * 2).astype(np.float32)
    dft = (tgt[:, :gamma] + rng.standard_normal((B, gamma, V))).astype(np.float32)
    toks = rng.integers(0, V, (B, gamma)).astype(np.int32)
    T = np.ones(B, np.float32)
    tgt[0, 1, 17] = np.nan
    tgt[1, 2, 5] = np.inf
    dft[2, 0, :] = -np.inf
    toks[3, 1] = V
    toks[4, 0] = -5
    T[5], T[6], T[7], T[8] = -1.0, np.nan, np.inf, 1e-8
    T[9] = 0.0
    dft[9, :, :] = np.nan                      # greedy never reads the draft
    tgt[10, :, ::3] = -np.inf                  # masked vocabulary
    dft[10, :, 1::3] = -np.inf
    T[11] = 0.0
    tgt[11, 0, :] = 1.0                        # all-tie greedy row: index 0 wins
    toks[11, 0] = 0
    tgt[12, 0, :] = -np.inf                    # all -inf row
    ua, ur = W.draw_uniforms(rng, (B, gamma)), W.draw_uniforms(rng, (B,))
    ua[14, 0] = 1.0                            # uniforms outside [0, 1): status 16
    ua[15, 1] = np.nan
    ur[16] = 1.0
    ur[17] = -0.5
    ua[18, :], ur[18] = 0.0, 0.0               # 0 is a valid uniform
    T[19], ua[19, 0], ur[19] = 0.0, 1.0, 2.0   # greedy reads no uniform
    for i, (lt, ld, x, u) in enumerate(vanished):
        b = 20 + i                             # the residual vanishes at position 0: status 8
        tgt[b, 0], dft[b, 0], toks[b, 0], ua[b, 0], ur[b] = lt, ld, x, 0.75, u
    w = W.Workload(f"edges-{V}", "f32", tgt, dft, toks, T, ua, ur)
    ref = oracle.verify_workload(w)
    assert ref.row_status[:9].tolist() == [2, 2, 2, 1, 1, 4, 4, 4, 4]
    assert ref.row_status[14:20].tolist() == [16, 16, 16, 16, 0, 0]
    assert (ref.row_status[20:] == 8).all() and (ref.n_accepted[20:] == 0).all()
    assert (ref.cdf_gap[20:] >= parity.BAND).all()   # compared exactly, status bit 8 included
    st = parity.compare(parity.run_gpu(w), ref)
    _report(f"edges-{V}", st)
    parity.assert_parity(st)


def test_golden_worked_example_gpu():
    import golden_cases
    fx, a = golden_cases.worked_example_v4()
    d = {k: torch.from_numpy(v).cuda() for k, v in a.items()}
    toks, n = binding.verify(**d)
    for i, c in enumerate(fx["cases"]):
        assert int(n[i]) == c["expect_n"], c["derivation"]
        assert toks[i].tolist() == c["expect_tokens"], c["derivation"]


@pytest.mark.parametrize("name", ["c2", "c3"])
def test_deterministic_and_workspace_reuse(name):
    """Same inputs -> identical outputs over repeated calls on one workspace."""
    w = W.make_workload(name)
    d = binding.to_device(w)
    first = [t.clone() for t in binding.verify(**d, return_log_norm=True)]
    for _ in range(5):
        again = binding.verify(**d, return_log_norm=True)
        for x, y in zip(first, again):
            assert torch.equal(x, y)


def test_generic_kernel_family():
    """The general two-kernel family, forced on shapes the streaming kernel takes."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, SPEC_VERIFY_FORCE_GENERIC="1")
    here = os.path.dirname(os.path.abspath(__file__))
    r = subprocess.run([sys.executable, os.path.join(here, "generic_path_check.py")], env=env,
                       capture_output=True, text=True, timeout=900)
    print(r.stdout[-3000:], r.stderr[-3000:])
    assert r.returncode == 0


def test_host_errors_leave_outputs_untouched():
    w = W.make_random(2, 2, 64, "f32", seed=5)
    d = binding.to_device(w)
    out = torch.full((2, 3), 123, dtype=torch.int32, device="cuda")
    n = torch.full((2,), 77, dtype=torch.int32, device="cuda")
    tiny = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(binding.SpecVerifyError):
        binding.verify(**d, out_tokens=out, out_n_accepted=n, workspace=tiny)
    torch.cuda.synchronize()
    assert (out == 123).all() and (n == 77).all()


def test_streams_and_graph_capture():
    """The call is stream-ordered and capturable in a CUDA graph."""
    w = W.make_workload("c1")
    d = binding.to_device(w)
    ref_t, ref_n = [t.clone() for t in binding.verify(**d)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        t2, n2 = binding.verify(**d)
    torch.cuda.current_stream().wait_stream(s)
    assert torch.equal(t2, ref_t) and torch.equal(n2, ref_n)
    out_t = torch.empty_like(ref_t)
    out_n = torch.empty_like(ref_n)
    g = torch.cuda.CUDAGraph()
    ws = binding.workspace_for(w.B, w.gamma, w.V, torch.float32, "cuda")
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        binding.verify(**d, out_tokens=out_t, out_n_accepted=out_n, workspace=ws)
    for _ in range(3):
        out_t.fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_t, ref_t) and torch.equal(out_n, ref_n)


@pytest.mark.parametrize("fill", [0xFF, 0x5A])
def test_workspace_needs_no_initialisation(fill):
    """A workspace filled with garbage and then shared by calls of different shapes,
    never re-zeroed: every call still matches the oracle (a call reads only what it
    wrote first; the general kernels' tickets are zeroed by the call's first launch)."""
    cases = [
        W.make_random(7, 4, 40008, "bf16", seed=5, T=np.array([0.0, 0.7, 1.0, 1.3] * 2, np.float32)[:7]),
        W.make_random(30, 2, 3001, "f32", seed=6, T=np.array([0.0, 0.9, 1.0] * 10, np.float32)),
        W.make_workload("c2"),
        W.make_random(7, 4, 40008, "bf16", seed=7, T=np.array([1.0] * 7, np.float32)),
    ]
    sizes = [binding.workspace_size(w.B, w.gamma, w.V, torch.bfloat16 if w.dtype == "bf16" else torch.float32)
             for w in cases]
    ws = torch.full((max(sizes),), fill, dtype=torch.uint8, device="cuda")
    for w in cases:
        d = binding.to_device(w)
        toks, n, ln, st = binding.verify(**d, return_log_norm=True, return_row_status=True, workspace=ws)
        torch.cuda.synchronize()
        g = dict(out_tokens=toks.cpu().numpy(), n_accepted=n.cpu().numpy(), log_norm=ln.cpu().numpy(),
                 row_status=st.cpu().numpy())
        stats = parity.compare(g, oracle.verify_workload(w))
        _report(f"garbage-{fill:#x}-{w.name}", stats)
        parity.assert_parity(stats)
