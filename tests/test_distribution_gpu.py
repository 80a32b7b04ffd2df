"""Distribution tests run directly on the GPU outputs (independent of the oracle):
emitted tokens follow the target distribution (chi-square and KS at 0.01 over
>= 10,000 trials per position), acceptance counts follow prod beta_i, the bonus
token follows p_gamma, and the oracle's cell-interior partition holds for the
GPU map as well."""
import numpy as np
import pytest
import torch

import oracle_pins as P
from speculative_decoding_verification_84_b200 import binding

pytestmark = pytest.mark.gpu


class _Res:
    pass


def gpu_verify(target, draft, draft_tokens, temperature, u_accept, u_resample, *, bf16=None, **_):
    """Adapter with the oracle's call signature, running the CUDA path."""
    tgt = torch.from_numpy(np.ascontiguousarray(target))
    dft = torch.from_numpy(np.ascontiguousarray(draft))
    if tgt.dtype == torch.uint16:
        tgt, dft = tgt.view(torch.bfloat16), dft.view(torch.bfloat16)
    dev = "cuda"
    toks, n, ln, st = binding.verify(
        tgt.to(dev), dft.to(dev), torch.from_numpy(np.ascontiguousarray(draft_tokens, np.int32)).to(dev),
        torch.from_numpy(np.ascontiguousarray(temperature, np.float32)).to(dev),
        torch.from_numpy(np.ascontiguousarray(u_accept, np.float32)).to(dev),
        torch.from_numpy(np.ascontiguousarray(u_resample, np.float32)).to(dev),
        return_log_norm=True, return_row_status=True)
    r = _Res()
    r.out_tokens, r.n_accepted = toks.cpu().numpy(), n.cpu().numpy()
    r.log_norm, r.row_status = ln.cpu().numpy(), st.cpu().numpy()
    return r


def test_gpu_distribution_ks_chi2():
    P.check_distribution(gpu_verify)


def test_gpu_bonus_distribution():
    P.check_bonus_distribution(gpu_verify)


def test_gpu_partition_cells():
    P.check_oracle_partition(gpu_verify)


def test_gpu_greedy_and_status_and_invariants():
    P.check_greedy_argmax(gpu_verify)
    P.check_status_edges(gpu_verify)
    P.check_output_invariants(gpu_verify)
