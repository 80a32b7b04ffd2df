"""spec_verify_noalloc: the entry point for callers that cannot allocate device
memory (an engine plugin's enqueue hook, a fixed memory budget owned by someone
else).  It must give the same results as spec_verify with a caller-owned
workspace, on consecutive calls that reuse its built-in scratch array.

This file is collected last on purpose, and it passes both alone in a fresh
process and after the other GPU tests."""
import ctypes

import numpy as np
import pytest
import torch

import parity
from speculative_decoding_verification_84_b200 import binding, workloads as W

pytestmark = pytest.mark.gpu

NOALLOC_SCRATCH_BYTES = 4 << 20


def _noalloc_fn():
    lib = binding.load_library()
    f = lib.spec_verify_noalloc
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [vp, vp, i32, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, vp, vp]
    f.restype = i32
    return f


def _call_noalloc(d, B, gamma, V, dt_code):
    f = _noalloc_fn()
    dev = d["target"].device
    out_t = torch.full((B, gamma + 1), -9, dtype=torch.int32, device=dev)
    out_n = torch.full((B,), -9, dtype=torch.int32, device=dev)
    ln = torch.empty((B, 2 * gamma + 1), dtype=torch.float64, device=dev)
    st = torch.empty((B,), dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream(dev)
    rc = f(d["target"].data_ptr(), d["draft"].data_ptr(), dt_code, d["draft_tokens"].data_ptr(),
           d["temperature"].data_ptr(), d["u_accept"].data_ptr(), d["u_resample"].data_ptr(),
           out_t.data_ptr(), out_n.data_ptr(), B, gamma, V, ln.data_ptr(), st.data_ptr(), s.cuda_stream)
    assert rc == 0, binding.status_string(rc)
    return out_t, out_n, ln, st


CASES = {
    "c2": lambda: W.make_workload("c2"),
    "c3": lambda: W.make_workload("c3"),
    "mixed": lambda: W.make_random(19, 6, 5003, "f32", seed=1234, T=([0.0, 0.8, 1.0, 1.3] * 5)[:19]),
    # the general kernels with a larger batch: its completion counters lie where the
    # previous call ("mixed") left its per-sequence records, so they start nonzero
    # unless the call clears them
    "mixed_wide_batch": lambda: W.make_random(300, 2, 1001, "bf16", seed=4321, T=([0.0, 0.7, 1.0] * 100)),
    # the streaming kernels with rows of more than 4096 tiles: tile sums in the
    # scratch rather than in shared memory
    "long_rows": lambda: W.make_random(2, 1, 600000, "f32", seed=99, T=[1.0, 0.8]),
}


@pytest.mark.parametrize("first,second", [("c2", "mixed"), ("c3", "c2"), ("mixed", "mixed_wide_batch"),
                                          ("long_rows", "mixed_wide_batch")])
def test_noalloc_matches_spec_verify_two_calls(first, second):
    for name in (first, second):                     # two calls in a row share the scratch
        w = CASES[name]()
        tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        assert binding.workspace_size(w.B, w.gamma, w.V, tdt) <= NOALLOC_SCRATCH_BYTES
        d = binding.to_device(w)
        ref_t, ref_n, ref_ln, ref_st = binding.verify(**d, return_log_norm=True, return_row_status=True)
        got_t, got_n, got_ln, got_st = _call_noalloc(d, w.B, w.gamma, w.V, binding._dt_code(tdt))
        torch.cuda.synchronize()
        assert torch.equal(got_t, ref_t), name
        assert torch.equal(got_n, ref_n), name
        assert torch.equal(got_st, ref_st), name
        a, b = got_ln.cpu().numpy(), ref_ln.cpu().numpy()
        fin = np.isfinite(b)
        assert (np.isfinite(a) == fin).all()
        assert np.all(np.abs(a[fin] - b[fin]) <= parity.LSE_RTOL * np.abs(b[fin])), name


def test_noalloc_rejects_oversized_shape():
    f = _noalloc_fn()
    B, gamma, V = 8192, 8, 151936                     # needs more than the built-in scratch
    assert binding.workspace_size(B, gamma, V, torch.bfloat16) > NOALLOC_SCRATCH_BYTES
    p = ctypes.c_void_p(1 << 20)                      # never dereferenced: rejected on the host
    rc = f(p, p, 1, p, p, p, p, p, p, B, gamma, V, None, None, None)
    assert rc == 4
