"""Run a few parity cases in a fresh process with SPEC_VERIFY_FORCE_GENERIC=1, so
the general kernel family is exercised on shapes the streaming kernel would take.
Exit status 0 when every case passes (used by test_parity_gpu.py)."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import parity  # noqa: E402
from speculative_decoding_verification_84_b200 import binding, workloads as W  # noqa: E402


def main():
    assert os.environ.get("SPEC_VERIFY_FORCE_GENERIC") == "1"
    import torch
    assert binding.kernels_per_call(64, 5, 128256, torch.bfloat16) == 3
    cases = [W.make_workload("c2"), W.make_workload("c3", seqs=range(16)),
             W.make_random(9, 3, 8192, "bf16", seed=77, T=np.array([0.0, 0.7, 1.0] * 3, np.float32)),
             W.make_workload("c5", B=600),
             W.make_random(33, 4, 200, "bf16", seed=78, T=np.array([0.0, 0.7, 1.0] * 11, np.float32))]
    for w in cases:
        st = parity.compare(parity.run_gpu(w), oracle.verify_workload(w))
        print(w.name, st)
        parity.assert_parity(st)
    print("generic path ok")


if __name__ == "__main__":
    main()
