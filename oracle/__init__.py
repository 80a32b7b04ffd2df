"""CPU oracle for batched speculative-sampling verification (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it, and this package imports
nothing from the product.

``verify`` wraps ``sv_oracle.c`` (plain C, double precision); see that file for
what is computed and which page passage each step follows.  ``build()``
compiles it with gcc into ``oracle/libsvoracle.so``.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sv_oracle.c")
_LIB = os.path.join(_HERE, "libsvoracle.so")

ST_TOKEN, ST_ROW, ST_TEMP, ST_RESID0, ST_UNIFORM, ST_TREE = 1, 2, 4, 8, 16, 32
RESIDUAL_MIN = 2.0 ** -18   # residual mass below this counts as vanished
NEAR_ACCEPT, NEAR_CDF = 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle (gcc -O2, OpenMP, strict IEEE: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def load_library(path: str):
    """Load an oracle shared library built from ``sv_oracle.c`` (or a test variant of it)."""
    lib = ctypes.CDLL(path)
    p = ctypes.c_void_p
    lib.sv_oracle_verify.argtypes = [p, p, ctypes.c_int, p, p, p, p, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_int, p, p, p, p, p, p, p,
                                     ctypes.c_int]
    lib.sv_oracle_verify.restype = ctypes.c_int
    lib.sv_oracle_max_threads.restype = ctypes.c_int
    lib.sv_oracle_fanout.argtypes = [ctypes.c_double, ctypes.c_int, ctypes.c_int, p]
    lib.sv_oracle_fanout.restype = ctypes.c_int
    lib.sv_oracle_topf.argtypes = [p, p, ctypes.c_int, p, ctypes.c_int, ctypes.c_int, ctypes.c_int, p, p, p,
                                   ctypes.c_int]
    lib.sv_oracle_topf.restype = ctypes.c_int
    lib.sv_oracle_cache_lookup.argtypes = [p, p, p, ctypes.c_int, ctypes.c_int, p, p]
    lib.sv_oracle_cache_lookup.restype = ctypes.c_int
    lib.sv_oracle_bandit_step.argtypes = [p, ctypes.c_int, ctypes.c_int, p, p, p, p, ctypes.c_int, ctypes.c_int,
                                          p, p]
    lib.sv_oracle_bandit_step.restype = ctypes.c_int
    lib.sv_oracle_bandit_simulate.argtypes = [p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, p, p, p]
    lib.sv_oracle_bandit_simulate.restype = ctypes.c_int
    lib.sv_oracle_tree_verify.argtypes = [p, p, ctypes.c_int, p, p, p, p, p, p, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, p, p, p, p, p, p, p, p, ctypes.c_int]
    lib.sv_oracle_tree_verify.restype = ctypes.c_int
    lib.sv_oracle_tree_prune.argtypes = [p, ctypes.c_int, p, p, p, ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, p, p]
    lib.sv_oracle_tree_prune.restype = ctypes.c_int
    lib.sv_oracle_gemm_bf16.argtypes = [p, p, ctypes.c_int, ctypes.c_int, ctypes.c_int, p]
    lib.sv_oracle_gemm_bf16.restype = ctypes.c_int
    lib.sv_oracle_lowrank_head.argtypes = [p, p, p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, p, p, p,
                                           p]
    lib.sv_oracle_lowrank_head.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = load_library(_LIB)
    return _lib


@dataclasses.dataclass
class OracleResult:
    out_tokens: np.ndarray   # [B, gamma+1] int32, -1 past the extra token
    n_accepted: np.ndarray   # [B] int32
    log_norm: np.ndarray     # [B, 2*gamma+1] float64 (target rows, then draft rows)
    row_status: np.ndarray   # [B] int32 bitmask
    near_tie: np.ndarray     # [B] int32 bitmask (1 accept test, 2 inverse CDF)
    accept_gap: np.ndarray   # [B] float64: min |log u_j - delta_j| over tested j
    cdf_gap: np.ndarray      # [B] float64: distance of u*S to the chosen bin's edges (probability
                             # units), or |S - RESIDUAL_MIN| after a rejection if smaller


def max_threads() -> int:
    return int(_load().sv_oracle_max_threads())


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def verify(target: np.ndarray, draft: np.ndarray, draft_tokens: np.ndarray,
           temperature: np.ndarray, u_accept: np.ndarray, u_resample: np.ndarray,
           *, bf16: bool | None = None, n_threads: int = 0, lib=None) -> OracleResult:
    """Run the oracle.  Logits are float32 arrays, or uint16 bf16 bit patterns."""
    lib = _load() if lib is None else lib
    target = np.ascontiguousarray(target)
    draft = np.ascontiguousarray(draft)
    if bf16 is None:
        bf16 = target.dtype == np.uint16
    want = np.uint16 if bf16 else np.float32
    if target.dtype != want or draft.dtype != want:
        raise TypeError("target/draft must both be float32 or both uint16 (bf16 bits)")
    B, g1, V = target.shape
    gamma = g1 - 1
    if draft.shape != (B, gamma, V):
        raise ValueError("draft shape must be [B, gamma, V]")
    toks = np.ascontiguousarray(draft_tokens, dtype=np.int32).reshape(B, gamma)
    T = np.ascontiguousarray(temperature, dtype=np.float32).reshape(B)
    ua = np.ascontiguousarray(u_accept, dtype=np.float32).reshape(B, gamma)
    ur = np.ascontiguousarray(u_resample, dtype=np.float32).reshape(B)
    out_t = np.empty((B, gamma + 1), dtype=np.int32)
    out_n = np.empty((B,), dtype=np.int32)
    ln = np.empty((B, 2 * gamma + 1), dtype=np.float64)
    st = np.empty((B,), dtype=np.int32)
    nr = np.empty((B,), dtype=np.int32)
    ag = np.empty((B,), dtype=np.float64)
    cg = np.empty((B,), dtype=np.float64)
    rc = lib.sv_oracle_verify(_ptr(target), _ptr(draft), int(bool(bf16)), _ptr(toks), _ptr(T),
                              _ptr(ua), _ptr(ur), B, gamma, V, _ptr(out_t), _ptr(out_n),
                              _ptr(ln), _ptr(st), _ptr(nr), _ptr(ag), _ptr(cg), int(n_threads))
    if rc != 0:
        raise RuntimeError(f"sv_oracle_verify failed ({rc})")
    return OracleResult(out_t, out_n, ln, st, nr, ag, cg)


def verify_workload(w, n_threads: int = 0) -> OracleResult:
    """Run the oracle on a ``Workload`` from the seeded generators."""
    return verify(w.target, w.draft, w.draft_tokens, w.temperature, w.u_accept, w.u_resample,
                  bf16=(w.dtype == "bf16"), n_threads=n_threads)


def fanout(alpha: float, gamma: int, budget: int, lib=None) -> np.ndarray:
    """Cache slots F_n per outcome n in [0, gamma]: geometric in n with acceptance
    rate alpha, summing to the budget (see ``sv_oracle.c``)."""
    lib = _load() if lib is None else lib
    F = np.empty((gamma + 1,), dtype=np.int32)
    if lib.sv_oracle_fanout(float(alpha), int(gamma), int(budget), _ptr(F)) != 0:
        raise ValueError("bad fan-out arguments")
    return F


def topf(target: np.ndarray, draft: np.ndarray, temperature: np.ndarray, F, *, bf16: bool | None = None,
         n_threads: int = 0, lib=None):
    """Top-F_n tokens of the extra token's distribution for every outcome n, and
    their probabilities: ([B, sum F] int32, [B, sum F] float64)."""
    lib = _load() if lib is None else lib
    target = np.ascontiguousarray(target)
    draft = np.ascontiguousarray(draft)
    if bf16 is None:
        bf16 = target.dtype == np.uint16
    B, g1, V = target.shape
    gamma = g1 - 1
    F = np.ascontiguousarray(F, dtype=np.int32).reshape(gamma + 1)
    T = np.ascontiguousarray(temperature, dtype=np.float32).reshape(B)
    Ft = int(F.sum())
    tok = np.empty((B, Ft), dtype=np.int32)
    prob = np.empty((B, Ft), dtype=np.float64)
    rc = lib.sv_oracle_topf(_ptr(target), _ptr(draft), int(bool(bf16)), _ptr(T), B, gamma, V, _ptr(F),
                            _ptr(tok), _ptr(prob), int(n_threads))
    if rc != 0:
        raise RuntimeError(f"sv_oracle_topf failed ({rc})")
    return tok, prob


def topf_workload(w, F, n_threads: int = 0):
    return topf(w.target, w.draft, w.temperature, F, bf16=(w.dtype == "bf16"), n_threads=n_threads)


def cache_lookup(out_tokens: np.ndarray, out_n: np.ndarray, cache: np.ndarray, F, lib=None) -> np.ndarray:
    """Slot of each sequence's outcome (n, extra token) in its cache, else -1."""
    lib = _load() if lib is None else lib
    out_tokens = np.ascontiguousarray(out_tokens, dtype=np.int32)
    B, g1 = out_tokens.shape
    gamma = g1 - 1
    out_n = np.ascontiguousarray(out_n, dtype=np.int32).reshape(B)
    F = np.ascontiguousarray(F, dtype=np.int32).reshape(gamma + 1)
    cache = np.ascontiguousarray(cache, dtype=np.int32).reshape(B, int(F.sum()))
    slot = np.empty((B,), dtype=np.int32)
    if lib.sv_oracle_cache_lookup(_ptr(out_tokens), _ptr(out_n), _ptr(cache), B, gamma, _ptr(F), _ptr(slot)) != 0:
        raise RuntimeError("sv_oracle_cache_lookup failed")
    return slot


BANDIT_UCB1, BANDIT_THOMPSON, BANDIT_THOMPSON_BETA = 0, 1, 2


class Bandit:
    """Host state of the draft-selection bandit (see ``sv_oracle.c``): t, the arm
    chosen last, N_k and R_k; ``step`` feeds one batch's n_accepted and returns the
    next arm."""

    def __init__(self, K: int, policy: int = BANDIT_UCB1, lib=None):
        self.K, self.policy = K, policy
        self.lib = _load() if lib is None else lib
        self.t = np.zeros(1, np.float64)
        self.arm = np.full(1, -1, np.int32)
        self.N = np.zeros(K, np.float64)
        self.R = np.zeros(K, np.float64)

    def step(self, n_accepted, gamma: int, u1=None, u2=None) -> int:
        n = np.ascontiguousarray(n_accepted, dtype=np.int32).reshape(-1)
        u1 = np.ascontiguousarray(np.zeros(self.K) if u1 is None else u1, dtype=np.float32)
        u2 = np.ascontiguousarray(np.zeros(self.K) if u2 is None else u2, dtype=np.float32)
        rc = self.lib.sv_oracle_bandit_step(_ptr(n), n.size, int(gamma), _ptr(self.t), _ptr(self.arm),
                                            _ptr(self.N), _ptr(self.R), self.K, self.policy, _ptr(u1), _ptr(u2))
        if rc != 0:
            raise ValueError("bad bandit arguments")
        return int(self.arm[0])


def bandit_simulate(mu, T: int, policy: int, uniforms: np.ndarray, lib=None, with_state: bool = False):
    """Regret of each run of the simulation (``sv_oracle_bandit_simulate``), and
    with ``with_state`` each run's final [t, arm, N, R]."""
    lib = _load() if lib is None else lib
    mu = np.ascontiguousarray(mu, dtype=np.float64).reshape(-1)
    K = mu.size
    uniforms = np.ascontiguousarray(uniforms, dtype=np.float32)
    runs = uniforms.shape[0]
    assert uniforms.shape == (runs, T + 1, 2 * K + 1)
    regret = np.empty(runs, np.float64)
    state = np.empty((runs, 2 + 2 * K), np.float64)
    if lib.sv_oracle_bandit_simulate(_ptr(mu), K, int(T), int(policy), runs, _ptr(uniforms), _ptr(regret),
                                     _ptr(state)) != 0:
        raise ValueError("bad bandit simulation arguments")
    return (regret, state) if with_state else regret


@dataclasses.dataclass
class TreeResult:
    out_nodes: np.ndarray    # [B, N] int32: accepted nodes in path order, then -1
    out_tokens: np.ndarray   # [B, N] int32: their tokens, the extra token, then -1
    n_accepted: np.ndarray   # [B] int32
    log_norm: np.ndarray     # [B, 2N] float64: target rows, then draft rows (NaN: not read)
    row_status: np.ndarray   # [B] int32
    near_tie: np.ndarray     # [B] int32 (1 accept test, 2 inverse CDF / fallback threshold)
    accept_gap: np.ndarray   # [B] float64
    cdf_gap: np.ndarray      # [B] float64


def tree_verify(target, draft, parent, tokens, temperature, u_accept, u_resample, keep=None, *,
                bf16: bool | None = None, n_threads: int = 0, lib=None) -> TreeResult:
    """Tree verification (``sv_oracle_tree_verify``): target, draft [B, N, V];
    parent, tokens, u_accept [B, N]; keep [B, N] or None."""
    lib = _load() if lib is None else lib
    target = np.ascontiguousarray(target)
    draft = np.ascontiguousarray(draft)
    if bf16 is None:
        bf16 = target.dtype == np.uint16
    B, N, V = target.shape
    assert draft.shape == (B, N, V)
    par = np.ascontiguousarray(parent, dtype=np.int32).reshape(B, N)
    tok = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, N)
    kp = None if keep is None else np.ascontiguousarray(keep, dtype=np.int32).reshape(B, N)
    T = np.ascontiguousarray(temperature, dtype=np.float32).reshape(B)
    ua = np.ascontiguousarray(u_accept, dtype=np.float32).reshape(B, N)
    ur = np.ascontiguousarray(u_resample, dtype=np.float32).reshape(B)
    r = TreeResult(np.empty((B, N), np.int32), np.empty((B, N), np.int32), np.empty(B, np.int32),
                   np.empty((B, 2 * N), np.float64), np.empty(B, np.int32), np.empty(B, np.int32),
                   np.empty(B, np.float64), np.empty(B, np.float64))
    rc = lib.sv_oracle_tree_verify(_ptr(target), _ptr(draft), int(bool(bf16)), _ptr(par), _ptr(tok),
                                   None if kp is None else _ptr(kp), _ptr(T), _ptr(ua), _ptr(ur), B, N, V,
                                   _ptr(r.out_nodes), _ptr(r.out_tokens), _ptr(r.n_accepted), _ptr(r.log_norm),
                                   _ptr(r.row_status), _ptr(r.near_tie), _ptr(r.accept_gap), _ptr(r.cdf_gap),
                                   int(n_threads))
    if rc != 0:
        raise RuntimeError(f"sv_oracle_tree_verify failed ({rc})")
    return r


def tree_prune(draft, parent, tokens, temperature, threshold: float, *, bf16: bool | None = None, lib=None):
    """Cumulative draft log-probability of every node and the nodes kept at
    ``threshold`` (``sv_oracle_tree_prune``): (keep [B, N] int32, cum [B, N])."""
    lib = _load() if lib is None else lib
    draft = np.ascontiguousarray(draft)
    if bf16 is None:
        bf16 = draft.dtype == np.uint16
    B, N, V = draft.shape
    par = np.ascontiguousarray(parent, dtype=np.int32).reshape(B, N)
    tok = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, N)
    T = np.ascontiguousarray(temperature, dtype=np.float32).reshape(B)
    keep = np.empty((B, N), np.int32)
    cum = np.empty((B, N), np.float64)
    if lib.sv_oracle_tree_prune(_ptr(draft), int(bool(bf16)), _ptr(par), _ptr(tok), _ptr(T), float(threshold),
                                B, N, V, _ptr(keep), _ptr(cum)) != 0:
        raise ValueError("bad tree shape")
    return keep, cum


def gemm_bf16(A, B, lib=None) -> np.ndarray:
    """A [M, K] @ B [N, K]^T over bf16 bit patterns (uint16), in fp64."""
    lib = _load() if lib is None else lib
    A = np.ascontiguousarray(A, dtype=np.uint16)
    B = np.ascontiguousarray(B, dtype=np.uint16)
    M, K = A.shape
    N = B.shape[0]
    assert B.shape == (N, K)
    out = np.empty((M, N), np.float64)
    if lib.sv_oracle_gemm_bf16(_ptr(A), _ptr(B), M, N, K, _ptr(out)) != 0:
        raise ValueError("bad shape")
    return out


def lowrank_head(h, w_down, w_up, temperature=None, lib=None):
    """The low-rank draft head (``sv_oracle_lowrank_head``): (u [M, r] bf16 bits,
    z [M, V] fp64, lse [M] of bf16(z) / T)."""
    lib = _load() if lib is None else lib
    h = np.ascontiguousarray(h, dtype=np.uint16)
    w_down = np.ascontiguousarray(w_down, dtype=np.uint16)
    w_up = np.ascontiguousarray(w_up, dtype=np.uint16)
    M, d = h.shape
    r = w_down.shape[0]
    V = w_up.shape[0]
    assert w_down.shape == (r, d) and w_up.shape == (V, r)
    T = None if temperature is None else np.ascontiguousarray(temperature, dtype=np.float32).reshape(M)
    u = np.empty((M, r), np.uint16)
    z = np.empty((M, V), np.float64)
    lse = np.empty(M, np.float64)
    if lib.sv_oracle_lowrank_head(_ptr(h), _ptr(w_down), _ptr(w_up), M, d, r, V, None if T is None else _ptr(T),
                                  _ptr(u), _ptr(z), _ptr(lse)) != 0:
        raise ValueError("bad shape")
    return u, z, lse
