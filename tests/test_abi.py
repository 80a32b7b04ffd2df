"""The C-ABI library loads and exports every function that include/*.h declares
(no GPU needed: nothing is called that touches the device)."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

from speculative_decoding_verification_84_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ ]*?[\s\*]+([a-z_][a-z0-9_]*)\s*\(",
                             text, flags=re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def test_header_declares_expected_api():
    assert set(binding.EXPORTED) <= _declared_functions()


def test_every_declared_symbol_is_exported(lib):
    for name in sorted(_declared_functions()):
        assert hasattr(lib, name), f"{name} missing from {build.LIB}"
        getattr(lib, name)  # resolves via dlsym


def test_nm_lists_symbols(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True, text=True).stdout
    for name in _declared_functions():
        assert re.search(rf"\bT {name}$", out, flags=re.M), name


def test_workspace_size_host_only(lib):
    s = binding.workspace_size(64, 5, 128256, __import__("torch").bfloat16)
    assert s > 0 and s % 256 == 0
    assert lib.spec_verify_workspace_size(0, 5, 100, 0) == 0
    assert lib.spec_verify_workspace_size(4, 0, 100, 0) == 0
    assert lib.spec_verify_workspace_size(4, 33, 100, 0) == 0
    assert lib.spec_verify_workspace_size(4, 2, 0, 0) == 0
    assert lib.spec_verify_workspace_size(4, 2, 100, 7) == 0
    # two launches per call on 16-byte-aligned rows of 4 KB or more (stream, draw), three
    # otherwise (ticket reset, row pass, resample), 0 on a bad shape
    assert lib.spec_verify_kernels_per_call(64, 5, 128256, 1) == 2
    assert lib.spec_verify_kernels_per_call(3, 2, 3001, 1) == 3
    assert lib.spec_verify_kernels_per_call(16384, 4, 64, 0) == 1
    assert lib.spec_verify_kernels_per_call(0, 2, 100, 0) == 0
    # a larger batch never needs less workspace
    sizes = [lib.spec_verify_workspace_size(b, 5, 128256, 1) for b in (1, 2, 64, 65, 256)]
    assert sizes == sorted(sizes)


def test_host_validation_before_launch(lib):
    """Host-checkable errors return before any CUDA call (safe without a GPU)."""
    vp = ctypes.c_void_p
    good = vp(1 << 20)
    ws_size = lib.spec_verify_workspace_size(2, 2, 64, 0)
    args = [good, good, 0, good, good, good, good, good, good, 2, 2, 64, good, ws_size, None, None, None]
    bad_dtype = list(args); bad_dtype[2] = 5
    assert lib.spec_verify(*bad_dtype) == 2
    bad_b = list(args); bad_b[9] = 0
    assert lib.spec_verify(*bad_b) == 1
    bad_g = list(args); bad_g[10] = 40
    assert lib.spec_verify(*bad_g) == 1
    null = list(args); null[0] = None
    assert lib.spec_verify(*null) == 1
    mis = list(args); mis[0] = vp((1 << 20) + 8)
    assert lib.spec_verify(*mis) == 3
    small = list(args); small[13] = ws_size - 1
    assert lib.spec_verify(*small) == 4
    for s in range(6):
        assert lib.spec_verify_status_string(s)


def test_fanout_host_matches_oracle(lib):
    """spec_verify_fanout runs on the host: it must allocate the slots exactly as
    the oracle's geometric rule (pinned in topf_pins.check_fanout_closed_forms)."""
    import numpy as np
    import oracle
    for alpha in (0.0, 0.1, 0.33, 0.5, 0.7, 0.95, 1.0):
        for gamma in (1, 4, 5, 8, 32):
            for budget in (0, 1, 3, 16, 64, 255):
                got = binding.fanout(alpha, gamma, budget)
                assert (got == oracle.fanout(alpha, gamma, budget)).all(), (alpha, gamma, budget)
    F = np.empty(3, np.int32)
    assert lib.spec_verify_fanout(1.5, 2, 4, F.ctypes.data) != 0
    assert lib.spec_verify_fanout(0.5, 0, 4, F.ctypes.data) != 0
    assert lib.spec_verify_fanout(0.5, 2, -1, F.ctypes.data) != 0


def test_bandit_host_validation(lib):
    """State size and the bandit entry points' host checks (no launch)."""
    vp = ctypes.c_void_p
    good = vp(1 << 20)
    assert lib.spec_verify_bandit_state_size(3) == 8 * 8
    assert lib.spec_verify_bandit_state_size(16) == 8 * 34
    assert lib.spec_verify_bandit_state_size(0) == 0 and lib.spec_verify_bandit_state_size(17) == 0
    assert lib.spec_verify_bandit_init(None, 3, None) == 1
    assert lib.spec_verify_bandit_init(good, 17, None) == 1
    assert lib.spec_verify_bandit_init(vp((1 << 20) + 4), 3, None) == 3
    step = [good, 4, 5, 0, None, None, good, 3, None, None]
    bad = list(step); bad[3] = 3                 # unknown policy
    assert lib.spec_verify_bandit_step(*bad) == 1
    bad = list(step); bad[3] = 1                 # Thompson sampling without uniforms
    assert lib.spec_verify_bandit_step(*bad) == 1
    bad = list(step); bad[2] = 0                 # gamma
    assert lib.spec_verify_bandit_step(*bad) == 1
    bad = list(step); bad[0] = None              # B > 0 without n_accepted
    assert lib.spec_verify_bandit_step(*bad) == 1
    bad = list(step); bad[6] = vp((1 << 20) + 4)  # state not 8-byte aligned
    assert lib.spec_verify_bandit_step(*bad) == 3
    sim = [good, 3, 100, 0, 4, good, good, None, None]
    bad = list(sim); bad[1] = 0
    assert lib.spec_verify_bandit_simulate(*bad) == 1
    bad = list(sim); bad[2] = -1
    assert lib.spec_verify_bandit_simulate(*bad) == 1
    bad = list(sim); bad[5] = None
    assert lib.spec_verify_bandit_simulate(*bad) == 1
    zero = list(sim); zero[4] = 0                # no runs: nothing to launch
    assert lib.spec_verify_bandit_simulate(*zero) == 0
