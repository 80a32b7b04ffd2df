"""Seeded synthetic inputs for batched speculative-sampling verification.

This module only draws random inputs.  It holds none of the verification
arithmetic (no normaliser, no acceptance test, no residual or bonus draw), so
both the CPU oracle and the CUDA path can be fed from it without sharing code.

The five workloads stand in for the pages' models and prompts, which are not
available here (TinyLlama / Llama-3 / Qwen logits on chat, code and maths
prompts; FlashSpec, "Resultados Principais"; SlimSpec, "Resultados").  Their
vocabulary sizes (32000, 128256, 151936) and speculation lengths (gamma 4-8)
follow those models' shapes:

  c1  B=1,     gamma=4, V=32000,  f32   target N(0,2^2); draft = target + N(0,0.5^2); T=1
  c2  B=8,     gamma=4, V=32000,  bf16  target N(0,3^2) with 50 distinct ids +6 per row;
                                        draft = target + N(0,1); T=0.7
  c3  B=64,    gamma=5, V=128256, bf16  target N(0,3^2) + Zipf(1.1) log-bias over a random
                                        permutation of ids; draft = rho*target +
                                        sqrt(1-rho^2)*N(0,3^2), rho=0.9; T=1
  c4  B=256,   gamma=8, V=151936, bf16  as c3, with rho in {0.6,0.8,0.95} and
                                        T in {0,0.6,1.0} by sequence index mod 3
  c5  B=16384, gamma=4, V=64,     f32   one (target, draft) pattern, both N(0,1.5^2)
                                        independent, replicated over all rows; T=1

Randomness.  Every bulky stream is seeded per sequence, so any subset of a
large batch can be regenerated on its own:
``SeedSequence(84 + config_index, spawn_key=(stream, b))`` with numpy PCG64.
Streams: 0 target noise, 1 per-row structure (c2 peaks), 2 draft noise,
3 Gumbel noise for drawing the draft tokens, and config-level streams
4 u_accept, 5 u_resample, 6 shared structure (c3/c4 permutation, c5 pattern).

Draft tokens are drawn from the draft distribution the verifier assumes,
softmax(draft_logits / T) on the *rounded* logits, with the Gumbel-max trick
(argmax of logits/T + Gumbel noise), or as the first argmax when T = 0.

Uniforms are exact float32 values (2k+1) * 2^-24 for k uniform in [0, 2^23),
so they lie strictly inside (0, 1) with spacing 2^-23.

bf16 values are produced by rounding the fp64 draw to fp32 and then to bf16
with round-to-nearest-even; arrays of bf16 are held as uint16 bit patterns.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

SEED_BASE = 84

CONFIGS = {
    "c1": dict(index=0, B=1, gamma=4, V=32000, dtype="f32"),
    "c2": dict(index=1, B=8, gamma=4, V=32000, dtype="bf16"),
    "c3": dict(index=2, B=64, gamma=5, V=128256, dtype="bf16"),
    "c4": dict(index=3, B=256, gamma=8, V=151936, dtype="bf16"),
    "c5": dict(index=4, B=16384, gamma=4, V=64, dtype="f32"),
}

_S_TARGET, _S_ROWSTRUCT, _S_DRAFT, _S_GUMBEL, _S_UACC, _S_URES, _S_SHARED = range(7)


@dataclasses.dataclass
class Workload:
    """One batch of verification inputs (host numpy arrays).

    target: [B, gamma+1, V] float32, or uint16 bf16 bit patterns when dtype == "bf16"
    draft:  [B, gamma, V]   same dtype as target
    draft_tokens: [B, gamma] int32
    temperature:  [B] float32 (0 = greedy)
    u_accept:     [B, gamma] float32 in (0, 1)
    u_resample:   [B] float32 in (0, 1)
    """

    name: str
    dtype: str
    target: np.ndarray
    draft: np.ndarray
    draft_tokens: np.ndarray
    temperature: np.ndarray
    u_accept: np.ndarray
    u_resample: np.ndarray

    @property
    def B(self) -> int:
        return self.target.shape[0]

    @property
    def gamma(self) -> int:
        return self.draft.shape[1]

    @property
    def V(self) -> int:
        return self.target.shape[2]

    def logits_as_f64(self, which: str) -> np.ndarray:
        """The exact stored logit values widened to float64."""
        a = self.target if which == "target" else self.draft
        if self.dtype == "bf16":
            return bf16_bits_to_f32(a).astype(np.float64)
        return a.astype(np.float64)

    def subset(self, idx: Sequence[int]) -> "Workload":
        idx = np.asarray(idx, dtype=np.int64)
        return Workload(self.name, self.dtype, np.ascontiguousarray(self.target[idx]),
                        np.ascontiguousarray(self.draft[idx]),
                        np.ascontiguousarray(self.draft_tokens[idx]),
                        np.ascontiguousarray(self.temperature[idx]),
                        np.ascontiguousarray(self.u_accept[idx]),
                        np.ascontiguousarray(self.u_resample[idx]))

    def logits_bytes(self) -> int:
        return self.target.nbytes + self.draft.nbytes


# ----------------------------------------------------------------------------- helpers

def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=tuple(key))))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); finite inputs."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _store(x64: np.ndarray, dtype: str) -> np.ndarray:
    x32 = x64.astype(np.float32)
    return f32_to_bf16_bits(x32) if dtype == "bf16" else x32


def _stored_to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    return (bf16_bits_to_f32(a) if dtype == "bf16" else a).astype(np.float64)


def uniforms_from_ints(k: np.ndarray) -> np.ndarray:
    """(2k+1) * 2^-24 as exact float32, for integers k in [0, 2^23)."""
    return ((2 * k.astype(np.int64) + 1).astype(np.float64) * 2.0 ** -24).astype(np.float32)


def draw_uniforms(rng: np.random.Generator, shape) -> np.ndarray:
    return uniforms_from_ints(rng.integers(0, 1 << 23, size=shape))


def gumbel_max_tokens(draft_f64: np.ndarray, T: float, gumbel_u: np.ndarray) -> np.ndarray:
    """Draw one token per row from softmax(row / T) via argmax(row/T + Gumbel); argmax if T == 0."""
    if T == 0.0:
        return np.argmax(draft_f64, axis=-1).astype(np.int32)
    g = -np.log(-np.log(gumbel_u))
    return np.argmax(draft_f64 / T + g, axis=-1).astype(np.int32)


def zipf_log_bias(V: int, perm: np.ndarray, exponent: float = 1.1) -> np.ndarray:
    """bias[perm[r-1]] = -exponent * ln r for ranks r = 1..V (log of Zipf weights r^-s)."""
    bias = np.empty(V, dtype=np.float64)
    bias[perm] = -exponent * np.log(np.arange(1, V + 1, dtype=np.float64))
    return bias


# ----------------------------------------------------------------------------- generator

def config_info(name: str) -> dict:
    return dict(CONFIGS[name])


def make_workload(name: str, *, seqs: Optional[Sequence[int]] = None, B: Optional[int] = None,
                  pattern: int = 0, seed: Optional[int] = None) -> Workload:
    """Generate config ``name`` (c1..c5).

    seqs:    optional subset of sequence indices to generate (streams are per sequence,
             so a subset equals the same rows of the full batch).
    B:       override the batch size (the first B sequences of an unbounded batch).
    pattern: for c5, which shared (target, draft) pattern to use (seed offset).
    seed:    override the base seed (default 84 + config index).
    """
    cfg = CONFIGS[name]
    gamma, V, dt = cfg["gamma"], cfg["V"], cfg["dtype"]
    B_full = cfg["B"] if B is None else int(B)
    base = (SEED_BASE + cfg["index"]) if seed is None else int(seed)
    if name == "c5":
        base += pattern
    idx = np.arange(B_full) if seqs is None else np.asarray(list(seqs), dtype=np.int64)
    n = len(idx)

    shared = _rng(base, _S_SHARED)
    perm = None
    pat_t = pat_d = None
    if name in ("c3", "c4"):
        perm = shared.permutation(V)
        bias = zipf_log_bias(V, perm)
    if name == "c5":
        pat_t = shared.standard_normal((gamma + 1, V)) * 1.5
        pat_d = shared.standard_normal((gamma, V)) * 1.5

    uacc_all = draw_uniforms(_rng(base, _S_UACC), (B_full, gamma))
    ures_all = draw_uniforms(_rng(base, _S_URES), (B_full,))

    tgt = np.empty((n, gamma + 1, V), dtype=np.uint16 if dt == "bf16" else np.float32)
    dft = np.empty((n, gamma, V), dtype=tgt.dtype)
    toks = np.empty((n, gamma), dtype=np.int32)
    temp = np.empty((n,), dtype=np.float32)

    for i, b in enumerate(idx):
        b = int(b)
        if name == "c1":
            T = 1.0
            t64 = _rng(base, _S_TARGET, b).standard_normal((gamma + 1, V)) * 2.0
            d64 = t64[:gamma] + _rng(base, _S_DRAFT, b).standard_normal((gamma, V)) * 0.5
        elif name == "c2":
            T = 0.7
            t64 = _rng(base, _S_TARGET, b).standard_normal((gamma + 1, V)) * 3.0
            rs = _rng(base, _S_ROWSTRUCT, b)
            for j in range(gamma + 1):
                t64[j, rs.choice(V, 50, replace=False)] += 6.0
            d64 = t64[:gamma] + _rng(base, _S_DRAFT, b).standard_normal((gamma, V)) * 1.0
        elif name in ("c3", "c4"):
            if name == "c3":
                T, rho = 1.0, 0.9
            else:
                T, rho = (0.0, 0.6, 1.0)[b % 3], (0.6, 0.8, 0.95)[b % 3]
            t64 = _rng(base, _S_TARGET, b).standard_normal((gamma + 1, V)) * 3.0 + bias
            d64 = rho * t64[:gamma] + math.sqrt(1.0 - rho * rho) * 3.0 * \
                _rng(base, _S_DRAFT, b).standard_normal((gamma, V))
        elif name == "c5":
            T = 1.0
            t64, d64 = pat_t, pat_d
        else:
            raise KeyError(name)
        tgt[i] = _store(t64, dt)
        dft[i] = _store(d64, dt)
        temp[i] = T
        gu = _rng(base, _S_GUMBEL, b).random((gamma, V))
        gu = np.clip(gu, 1e-300, 1.0 - 2.0 ** -53)
        toks[i] = gumbel_max_tokens(_stored_to_f64(dft[i], dt), T, gu)

    return Workload(name, dt, tgt, dft, toks, temp, np.ascontiguousarray(uacc_all[idx]),
                    np.ascontiguousarray(ures_all[idx]))


def make_random(B: int, gamma: int, V: int, dtype: str, *, seed: int, T=1.0,
                target_sd: float = 2.0, draft_noise: float = 1.0) -> Workload:
    """A small random batch of any shape (for ragged-size and property tests).

    T may be a scalar or a length-B sequence.  Draft = target + N(0, draft_noise^2)."""
    rng = _rng(seed, 99)
    t64 = rng.standard_normal((B, gamma + 1, V)) * target_sd
    d64 = t64[:, :gamma] + rng.standard_normal((B, gamma, V)) * draft_noise
    temp = np.broadcast_to(np.asarray(T, dtype=np.float32), (B,)).copy()
    tgt, dft = _store(t64, dtype), _store(d64, dtype)
    toks = np.empty((B, gamma), dtype=np.int32)
    gu = np.clip(rng.random((B, gamma, V)), 1e-300, 1.0 - 2.0 ** -53)
    for b in range(B):
        toks[b] = gumbel_max_tokens(_stored_to_f64(dft[b], dtype), float(temp[b]), gu[b])
    return Workload(f"random_{B}x{gamma}x{V}_{dtype}", dtype, tgt, dft, toks, temp,
                    draw_uniforms(rng, (B, gamma)), draw_uniforms(rng, (B,)))


def bandit_uniforms(runs: int, T: int, K: int, seed: int) -> np.ndarray:
    """Uniforms of the draft-selection regret simulation: [runs][T + 1][2K + 1]
    float32 in (0, 1), row s holding step s's u1 (K values) and u2 (K values),
    then round s's reward draw.  Each run is seeded on its own (stream 7, key run)."""
    out = np.empty((runs, T + 1, 2 * K + 1), np.float32)
    for r in range(runs):
        out[r] = draw_uniforms(_rng(seed, 7, r), (T + 1, 2 * K + 1))
    return out


# ----------------------------------------------------------------------------- token trees

@dataclasses.dataclass
class TreeWorkload:
    """One batch of tree-verification inputs (host numpy arrays).

    target, draft: [B, N, V] (float32, or uint16 bf16 bits): the next-token logits
    at node i's context; parent, tokens, u_accept: [B, N] (node 0 is the root:
    parent -1, token and uniform unused); temperature, u_resample: [B]."""

    name: str
    dtype: str
    target: np.ndarray
    draft: np.ndarray
    parent: np.ndarray
    tokens: np.ndarray
    temperature: np.ndarray
    u_accept: np.ndarray
    u_resample: np.ndarray

    @property
    def B(self):
        return self.target.shape[0]

    @property
    def N(self):
        return self.target.shape[1]

    @property
    def V(self):
        return self.target.shape[2]


def tree_parents(branching: Sequence[int]) -> np.ndarray:
    """Parent array of a tree in breadth-first order: the root has branching[0]
    children, each of those branching[1], and so on (so parent[i] < i)."""
    par, level = [-1], [0]
    for k in branching:
        nxt = []
        for p in level:
            for _ in range(int(k)):
                par.append(p)
                nxt.append(len(par) - 1)
        level = nxt
    return np.asarray(par, dtype=np.int32)


def make_tree(B: int, branching: Sequence[int], V: int, dtype: str, *, seed: int, T=1.0, rho: float = 0.9,
              name: Optional[str] = None) -> TreeWorkload:
    """A batch of token trees of one shape, built like c3: every node's target
    row N(0, 3^2) + a Zipf(1.1) log-bias over a permutation shared by the batch,
    its draft row rho * target + sqrt(1 - rho^2) * N(0, 3^2).  Node i's token is
    drawn from softmax(draft row of its parent / T) (T = 1 for greedy sequences,
    so siblings differ), independently for every sibling.  T may be a scalar or
    a sequence, repeated over the batch.  Each sequence has its own streams (key
    8, b)."""
    par = tree_parents(branching)
    N = par.size
    temp = np.resize(np.asarray(T, dtype=np.float32).reshape(-1), B).astype(np.float32)
    bias = zipf_log_bias(V, _rng(seed, 8, 1 << 20).permutation(V))
    dt = np.uint16 if dtype == "bf16" else np.float32
    tgt = np.empty((B, N, V), dt)
    dft = np.empty((B, N, V), dt)
    tok = np.zeros((B, N), np.int32)
    for b in range(B):
        rng = _rng(seed, 8, b)
        t64 = rng.standard_normal((N, V)) * 3.0 + bias
        d64 = rho * t64 + math.sqrt(1.0 - rho * rho) * 3.0 * rng.standard_normal((N, V))
        tgt[b] = _store(t64, dtype)
        dft[b] = _store(d64, dtype)
        dstored = _stored_to_f64(dft[b], dtype)
        Tb = float(temp[b]) if temp[b] > 0 else 1.0
        gu = np.clip(rng.random((N, V)), 1e-300, 1.0 - 2.0 ** -53)
        for i in range(1, N):
            tok[b, i] = gumbel_max_tokens(dstored[par[i]][None], Tb, gu[i][None])[0]
    urng = _rng(seed, 8, (1 << 20) + 1)
    ua = draw_uniforms(urng, (B, N))
    ur = draw_uniforms(urng, (B,))
    label = name or f"tree_{B}x{'-'.join(map(str, branching))}x{V}_{dtype}"
    return TreeWorkload(label, dtype, tgt, dft, np.tile(par, (B, 1)), tok, temp, ua, ur)


# ----------------------------------------------------------------------------- low-rank draft head

@dataclasses.dataclass
class LowRankWorkload:
    """Inputs of the low-rank draft head z = W_up (W_down h), as bf16 bit
    patterns: h [M, d], w_down [r, d], w_up [V, r]; temperature [M] (the draft
    position's sequence temperature)."""

    name: str
    h: np.ndarray
    w_down: np.ndarray
    w_up: np.ndarray
    temperature: np.ndarray


def make_lowrank(M: int, d: int, r: int, V: int, *, seed: int, scale: float = 3.0, T=1.0,
                 name: Optional[str] = None) -> LowRankWorkload:
    """Random-initialised head (no trained weights here): h ~ N(0, 1),
    W_down ~ N(0, 1/d), W_up ~ N(0, scale^2 / r), so u = W_down h has unit variance
    and the logits z have standard deviation about ``scale`` (3, as the target
    logits of c3).  T may be a scalar or a sequence, repeated over the rows."""
    rng = _rng(seed, 9)
    h = f32_to_bf16_bits(rng.standard_normal((M, d)).astype(np.float32))
    wd = f32_to_bf16_bits((rng.standard_normal((r, d)) / math.sqrt(d)).astype(np.float32))
    wu = f32_to_bf16_bits((rng.standard_normal((V, r)) * (scale / math.sqrt(r))).astype(np.float32))
    temp = np.resize(np.asarray(T, dtype=np.float32).reshape(-1), M).astype(np.float32)
    return LowRankWorkload(name or f"lowrank_{M}x{d}x{r}x{V}", h, wd, wu, temp)
