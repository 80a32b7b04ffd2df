"""Build the CUDA C-ABI library in-tree with nvcc for sm_100a.

    python -m speculative_decoding_verification_84_b200.build

produces ``speculative_decoding_verification_84_b200/lib/libspecverify.so``
from ``csrc/spec_verify.cu`` and the public header ``include/spec_verify.h``.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "spec_verify.cu")
DEPS = [os.path.join(HERE, "csrc", f)
        for f in ("sv_common.cuh", "sv_generic.cuh", "sv_pass.cuh", "sv_small.cuh", "sv_topf.cuh", "sv_bandit.cuh",
                  "sv_tree.cuh", "sv_lowrank.cuh")]
HEADER = os.path.join(ROOT, "include", "spec_verify.h")
LIB_DIR = os.path.join(HERE, "lib")
LIB = os.path.join(LIB_DIR, "libspecverify.so")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(LIB_DIR, exist_ok=True)
    newest = max(os.path.getmtime(f) for f in [SRC, HEADER, *DEPS])
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-o", tmp, SRC]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
