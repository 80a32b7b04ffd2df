"""Pins of the oracle's low-rank draft head (SlimSpec, Metodologia, "Arquitetura":
z = W_up W_down h), each against something other than the oracle itself: numpy
float64 matrix products, bf16 rounding done with integer arithmetic on the
float64 bits, exact integer associativity, closed-form log-normalisers and
hand-worked rounding ties.  Every check takes an object ``O`` with ``gemm_bf16``
and ``lowrank_head`` (the oracle module or a stand-in with a planted mistake)."""
from __future__ import annotations

import math
import struct

import numpy as np

from speculative_decoding_verification_84_b200 import workloads as W


def bf16_rne_bits(x: float) -> int:
    """bf16 bit pattern of the nearest bf16 value to the float64 x (ties to even),
    by integer arithmetic on the float64 bit pattern (normal range only)."""
    b = struct.unpack("<Q", struct.pack("<d", x))[0]
    sign = b >> 63
    e = (b >> 52) & 0x7FF
    mant = b & ((1 << 52) - 1)
    assert 0 < e < 0x7FF and (e - 1023) >= -126, x
    full = (1 << 52) | mant          # 53 significant bits
    keep = full >> 45                # 8 significant bits
    rest = full & ((1 << 45) - 1)
    half = 1 << 44
    if rest > half or (rest == half and (keep & 1)):
        keep += 1
    if keep == 1 << 8:               # carried into the next binade
        keep >>= 1
        e += 1
    exp32 = e - 1023 + 127
    return (sign << 15) | (exp32 << 7) | (keep & 0x7F)


def _bits_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _f32_to_bits(x):
    return W.f32_to_bf16_bits(np.asarray(x, np.float32))


def check_gemm_numpy(O):
    """gemm_bf16 equals numpy's float64 product of the widened inputs (the products
    are exact in float64; only the summation order differs)."""
    rng = np.random.default_rng(1)
    for M, N, K in [(1, 1, 1), (5, 7, 3), (17, 9, 64), (3, 40, 200)]:
        A = _f32_to_bits(rng.standard_normal((M, K)))
        B = _f32_to_bits(rng.standard_normal((N, K)))
        want = _bits_to_f64(A) @ _bits_to_f64(B).T
        got = O.gemm_bf16(A, B)
        assert np.allclose(got, want, rtol=1e-13, atol=1e-13), (M, N, K)
    A = _f32_to_bits([[1.0, 2.0]])
    B = _f32_to_bits([[3.0, 0.0], [0.0, 5.0]])
    assert O.gemm_bf16(A, B).tolist() == [[3.0, 10.0]]   # B's rows, not its columns


def check_u_rounding(O):
    """u = bf16(W_down h) with ties to even: hand-worked ties (1 + 2^-8 -> 1;
    1 + 2^-7 + 2^-8 -> 1 + 2^-6; -(1 + 2^-8) -> -1), and on random inputs the
    bits from integer rounding of numpy's float64 sums."""
    cases = [([1.0, 2.0 ** -8], 1.0), ([1.0 + 2.0 ** -7, 2.0 ** -8], 1.0 + 2.0 ** -6),
             ([-1.0, -(2.0 ** -8)], -1.0), ([3.0, 2.0 ** -7], 3.0), ([1.0, 2.0 ** -8 + 2.0 ** -12], 1.0 + 2.0 ** -7)]
    for hv, want in cases:
        h = _f32_to_bits([hv])
        wd = _f32_to_bits([[1.0, 1.0]])
        wu = _f32_to_bits([[1.0]])
        u, z, _ = O.lowrank_head(h, wd, wu)
        assert _bits_to_f64(u)[0, 0] == want, (hv, _bits_to_f64(u)[0, 0], want)
        assert z[0, 0] == want
    rng = np.random.default_rng(2)
    M, d, r = 6, 50, 9
    h = _f32_to_bits(rng.standard_normal((M, d)))
    wd = _f32_to_bits(rng.standard_normal((r, d)) * 0.2)
    wu = _f32_to_bits(rng.standard_normal((4, r)))
    u, _, _ = O.lowrank_head(h, wd, wu)
    exact = _bits_to_f64(h) @ _bits_to_f64(wd).T
    want = np.array([[bf16_rne_bits(float(x)) for x in row] for row in exact], np.uint16)
    assert (u == want).all()


def check_exact_associativity(O):
    """Small integers: every sum is exact and u fits bf16 exactly, so
    z = W_up (W_down h) = (W_up W_down) h in exact integer arithmetic."""
    rng = np.random.default_rng(3)
    M, d, r, V = 4, 12, 5, 30
    hi = rng.integers(-3, 4, size=(M, d))
    wdi = rng.integers(-2, 3, size=(r, d))
    wui = rng.integers(-3, 4, size=(V, r))
    u_int = hi @ wdi.T
    assert np.abs(u_int).max() < 256          # exact in bf16's 8 significant bits
    u, z, _ = O.lowrank_head(_f32_to_bits(hi), _f32_to_bits(wdi), _f32_to_bits(wui))
    assert (_bits_to_f64(u) == u_int).all()
    assert (z == hi @ (wui @ wdi).T).all()


def check_lse(O):
    """lse of the bf16 logits: constant logits c give c/T + ln V; on random heads it
    equals math.fsum's log-sum-exp of the integer-rounded bf16(z); T = 0 gives NaN."""
    V = 37
    for c, T in [(2.0, 1.0), (-3.0, 0.5), (0.0, 2.0)]:
        h = _f32_to_bits([[1.0]])
        wd = _f32_to_bits([[1.0]])
        wu = _f32_to_bits(np.full((V, 1), c))
        _, _, lse = O.lowrank_head(h, wd, wu, [T])
        assert abs(lse[0] - (c / T + math.log(V))) < 1e-12, (c, T, lse[0])
    w = W.make_lowrank(3, 40, 8, 300, seed=4, T=[1.0, 0.7, 0.0])
    _, z, lse = O.lowrank_head(w.h, w.w_down, w.w_up, w.temperature)
    for m in range(3):
        T = float(w.temperature[m])
        if T == 0.0:
            assert math.isnan(lse[m])
            continue
        zr = [float(_bits_to_f64([bf16_rne_bits(float(x))])[0]) for x in z[m]]
        mx = max(zr)
        want = mx / T + math.log(math.fsum(math.exp((x - mx) / T) for x in zr))
        assert abs(lse[m] - want) < 1e-12 * max(1.0, abs(want)), (m, lse[m], want)


ALL_LOWRANK_CHECKS = [check_gemm_numpy, check_u_rounding, check_exact_associativity, check_lse]
