"""Compile libstepq.so (CUDA for sm_100a) in-tree with nvcc.

    python -m quantized_recurrent_state_b200.build [--force]

Flags: -gencode arch=compute_100a,code=sm_100a -lineinfo -O3 --fmad=false
(no multiply-add contraction: every fp32 operation rounds where the
arithmetic definition says it does; explicit fma() calls stay fused), host
code with -ffp-contract=off.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libstepq.so")
SOURCES = ["stepq_api.cu", "stepq_step.cu", "stepq_head.cu", "stepq_head_tm.cu", "stepq_aux.cu", "stepq_prefill.cu", "stepq_prefill_tc.cu", "stepq_tc_selftest.cu"]
HEADERS = ["stepq_dev.cuh", "stepq_pipe.cuh", "stepq_head.cuh", "stepq_prefill.cuh", "stepq_tc.cuh", os.path.join("..", "..", "include", "stepq.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def nvcc_cmd(out: str, extra=()):
    return [NVCC, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            "--fmad=false", "-Xcompiler", "-fPIC,-ffp-contract=off", "-shared", "-o", out,
            *[os.path.join(CSRC, s) for s in SOURCES], *extra]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or _stale():
        tmp = LIB + ".tmp"
        cmd = nvcc_cmd(tmp, ["-Xptxas", "-v"] if verbose else [])
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
