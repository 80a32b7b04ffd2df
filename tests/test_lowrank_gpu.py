"""GPU parity of the low-rank draft head (SlimSpec, Metodologia, "Arquitetura":
z = W_up W_down h) on the tensor cores, through the C ABI, against the fp64
oracle.

Tolerances, from the arithmetic: the kernel rounds an fp32 accumulation of
exact bf16 products to bf16, the oracle sums in fp64.  So every output is within
one bf16 rounding of the exact sum plus the fp32 accumulation error:
|out - exact| <= 2^-8 |exact| + 2^-14 * sum_k |a_k b_k| (the second term bounds
K fp32 roundings with a wide margin), and almost all outputs equal the oracle's
own bf16 rounding (at least 98 %: a difference needs the exact sum within the
tiny fp32 error of a bf16 rounding boundary).  The row normaliser of up(u), fed
the oracle's own bf16 intermediate, is within sum_v p_v ulp(z_v) / T + 1e-6 of the
oracle's (each logit at most one bf16 ulp away), and within 1e-6 relative of
spec_verify's normaliser of the same logits (the same arithmetic on the same
bf16 values)."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_84_b200 import binding, workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _f(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _abs_bits(b):
    return (np.asarray(b, np.uint16) & 0x7FFF).astype(np.uint16)


def _bf16_ulp(x):
    x = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def _check_gemm(got_bits, exact, absum):
    got = _f(got_bits)
    assert np.all(np.abs(got - exact) <= 2.0 ** -8 * np.abs(exact) + 2.0 ** -14 * absum + 1e-30)
    assert (got_bits == _rne_bits(exact)).mean() >= 0.98


def _rne_bits(x):
    """bf16 bits of float64 values, ties to even, by integer arithmetic on the bits
    (normal range; zeros map to signed zeros)."""
    b = np.asarray(x, np.float64).view(np.uint64)
    sign = (b >> np.uint64(63)).astype(np.uint64)
    e = ((b >> np.uint64(52)) & np.uint64(0x7FF)).astype(np.int64)
    mant = (b & np.uint64((1 << 52) - 1)) | np.uint64(1 << 52)
    keep = (mant >> np.uint64(45)).astype(np.int64)
    rest = (mant & np.uint64((1 << 45) - 1)).astype(np.int64)
    half = 1 << 44
    up = (rest > half) | ((rest == half) & ((keep & 1) == 1))
    keep = keep + up
    carry = keep == (1 << 8)
    keep = np.where(carry, keep >> 1, keep)
    e = np.where(carry, e + 1, e)
    exp32 = e - 1023 + 127
    bits = (sign.astype(np.int64) << 15) | (exp32 << 7) | (keep & 0x7F)
    bits = np.where(e == 0, sign.astype(np.int64) << 15, bits)
    return bits.astype(np.uint16)


@pytest.mark.parametrize("M,d,r,V", [(200, 256, 64, 1000), (1, 8, 8, 1), (127, 72, 40, 33), (129, 256, 136, 4104),
                                     (64, 512, 96, 255), (257, 128, 64, 32000)])
def test_lowrank_shapes(M, d, r, V):
    """Ragged rows (partial 128-row tiles), K not a multiple of 64 (zero-filled
    tails), V not a multiple of 8 or of 256 (scalar stores, partial column tiles)."""
    w = W.make_lowrank(M, d, r, V, seed=M + d + r + V, T=[1.0, 0.7, 0.0, 2.0])
    dv = binding.lowrank_to_device(w, DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    u = binding.lowrank_down(dv["h"], dv["w_down"], error=err)
    uo, zo, lo = oracle.lowrank_head(w.h, w.w_down, w.w_up, w.temperature)
    u_exact = oracle.gemm_bf16(w.h, w.w_down)
    _check_gemm(_bits(u), u_exact, oracle.gemm_bf16(_abs_bits(w.h), _abs_bits(w.w_down)))
    # the second contraction from the oracle's own intermediate
    z, lse = binding.lowrank_up(torch.from_numpy(uo).view(torch.bfloat16).to(DEV), dv["w_up"], dv["temperature"],
                                error=err)
    _check_gemm(_bits(z), zo, oracle.gemm_bf16(_abs_bits(uo), _abs_bits(w.w_up)))
    lse = lse.cpu().numpy()
    for m in range(M):
        T = float(w.temperature[m])
        if T == 0.0:
            assert np.isnan(lse[m]) and np.isnan(lo[m])
            continue
        zr = _f(_rne_bits(zo[m]))
        p = np.exp((zr - zr.max()) / T)
        p /= p.sum()
        bound = float(np.sum(p * _bf16_ulp(zr))) / T + 1e-6
        assert abs(lse[m] - lo[m]) <= bound, (m, lse[m], lo[m], bound)
    # the whole head
    z2, l2 = binding.lowrank_head(dv["h"], dv["w_down"], dv["w_up"], dv["temperature"], error=err)
    absz = oracle.gemm_bf16(_abs_bits(uo), _abs_bits(w.w_up))
    # u may differ from the oracle's by one bf16 ulp per element: widen by W_up |ulp(u)|
    du = oracle.gemm_bf16(_rne_bits(_bf16_ulp(_f(uo))), _abs_bits(w.w_up))
    got = _f(_bits(z2))
    assert np.all(np.abs(got - zo) <= 2.0 ** -8 * np.abs(zo) + 2.0 ** -14 * absz + 1.01 * du + 1e-30)
    assert int(err.item()) == 0


def test_lowrank_h3_sampled():
    """The bench workload (M = 320 draft positions = 64 sequences x gamma 5, d = 4096,
    r = d/8 = 512, V = 128256): the whole down contraction, and the up contraction
    and normalisers of 6 sampled rows over the full vocabulary."""
    w = W.make_lowrank(320, 4096, 512, 128256, seed=2005, T=1.0)
    dv = binding.lowrank_to_device(w, DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    z, lse = binding.lowrank_head(dv["h"], dv["w_down"], dv["w_up"], dv["temperature"], error=err)
    u = binding.lowrank_down(dv["h"], dv["w_down"], error=err)
    _check_gemm(_bits(u), oracle.gemm_bf16(w.h, w.w_down), oracle.gemm_bf16(_abs_bits(w.h), _abs_bits(w.w_down)))
    rows = [0, 1, 127, 128, 255, 319]
    uo, zo, lo = oracle.lowrank_head(w.h[rows], w.w_down, w.w_up, w.temperature[rows])
    zr, _ = binding.lowrank_up(torch.from_numpy(uo).view(torch.bfloat16).to(DEV), dv["w_up"],
                               dv["temperature"][rows].contiguous(), error=err)
    _check_gemm(_bits(zr), zo, oracle.gemm_bf16(_abs_bits(uo), _abs_bits(w.w_up)))
    got = _f(_bits(z))[rows]
    du = oracle.gemm_bf16(_rne_bits(_bf16_ulp(_f(uo))), _abs_bits(w.w_up))
    absz = oracle.gemm_bf16(_abs_bits(uo), _abs_bits(w.w_up))
    assert np.all(np.abs(got - zo) <= 2.0 ** -8 * np.abs(zo) + 2.0 ** -14 * absz + 1.01 * du + 1e-30)
    assert int(err.item()) == 0


def test_lowrank_lse_matches_spec_verify():
    """The fused normaliser equals spec_verify's out_log_norm of the same draft rows
    (both GPU, same bf16 logits, same arithmetic): within 1e-6 relative."""
    B, gamma, V = 8, 4, 32000
    w = W.make_lowrank(B * gamma, 256, 64, V, seed=11, T=np.repeat([1.0, 0.7, 1.3, 1.0, 0.5, 1.0, 2.0, 1.0], gamma))
    dv = binding.lowrank_to_device(w, DEV)
    z, lse = binding.lowrank_head(dv["h"], dv["w_down"], dv["w_up"], dv["temperature"])
    draft = z.view(B, gamma, V).contiguous()
    target = torch.cat([draft, draft[:, :1]], 1).contiguous()
    T = dv["temperature"].view(B, gamma)[:, 0].contiguous()
    tok = torch.zeros((B, gamma), dtype=torch.int32, device=DEV)
    ua = torch.full((B, gamma), 0.5, device=DEV)
    ur = torch.full((B,), 0.5, device=DEV)
    _, _, ln = binding.verify(target, draft, tok, T, ua, ur, return_log_norm=True)
    sv_lse = ln[:, gamma + 1:].reshape(-1).cpu().numpy()
    got = lse.cpu().numpy()
    assert np.allclose(got, sv_lse, rtol=1e-6, atol=1e-6), np.max(np.abs(got - sv_lse))
