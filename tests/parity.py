"""GPU-vs-oracle comparison used by the GPU parity tests.

Decisions: n_accepted and out_tokens must be bit-exact, except for sequences the
oracle reports within 1e-6 of a decision boundary (|log u - delta| or the
inverse-CDF gap); those are counted, and mismatches among them reported.
Normalisers: |gpu - oracle| <= 1e-5 * |oracle| per row, NaN pattern equal.
Row status: exact, except bit 8 (residual vanished) of a near-tie sequence: that
bit records the outcome of the same rounding-level decision."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from speculative_decoding_verification_84_b200 import binding

BAND = 1e-6
LSE_RTOL = 1e-5


def run_gpu(w, device="cuda"):
    d = binding.to_device(w, device)
    toks, n, ln, st = binding.verify(**d, return_log_norm=True, return_row_status=True)
    torch.cuda.synchronize()
    return dict(out_tokens=toks.cpu().numpy(), n_accepted=n.cpu().numpy(), log_norm=ln.cpu().numpy(),
                row_status=st.cpu().numpy())


def _status_view(st, near):
    st = np.asarray(st)
    return np.where(near, st & ~oracle.ST_RESID0, st)


def compare(gpu: dict, ref: oracle.OracleResult, idx=None) -> dict:
    """Compare GPU outputs (optionally rows ``idx`` of them) with the oracle's."""
    g = {k: (v if idx is None else v[idx]) for k, v in gpu.items()}
    near = (ref.accept_gap < BAND) | (ref.cdf_gap < BAND)
    same = (g["n_accepted"] == ref.n_accepted) & (g["out_tokens"] == ref.out_tokens).all(axis=1)
    bad = ~same & ~near
    fin = np.isfinite(ref.log_norm)
    lse_ok = (np.isfinite(g["log_norm"]) == fin).all()
    rel = np.abs(g["log_norm"][fin] - ref.log_norm[fin]) / np.maximum(np.abs(ref.log_norm[fin]), 1e-300)
    stats = dict(B=len(same), exact=int(same.sum()), near=int(near.sum()),
                 near_mismatch=int((~same & near).sum()), mismatch=int(bad.sum()),
                 mismatch_rows=np.nonzero(bad)[0][:10].tolist(),
                 lse_max_rel=float(rel.max()) if rel.size else 0.0, lse_nan_pattern_ok=bool(lse_ok),
                 status_ok=bool((_status_view(g["row_status"], near) == _status_view(ref.row_status, near)).all()))
    return stats


def assert_parity(stats: dict):
    assert stats["mismatch"] == 0, stats
    assert stats["lse_nan_pattern_ok"], stats
    assert stats["lse_max_rel"] <= LSE_RTOL, stats
    assert stats["status_ok"], stats
