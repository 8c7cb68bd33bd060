"""Build libjolt.so (the sm_100a C-ABI library) in-tree with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libjolt.so")
SOURCES = ["jolt_api.cu"]
DEPS = ["jolt_api.cu", "common.cuh", "gemm.cuh", "kernels.cuh", "misc.cuh", "umma.cuh", "eig_cluster.cuh", "chol.cuh",
        "fp16_exact.cuh", "table_tc.cuh", "attend.cuh", "eig_large.cuh"]


def nvcc_cmd(out: str = LIB, extra=()) -> list:
    return (["nvcc", "-std=c++17", "-O3", "-lineinfo",
             "-gencode", "arch=compute_100a,code=sm_100a",
             "-Xcompiler", "-fPIC", "-shared",
             "-I", os.path.join(ROOT, "include"),
             "-o", out] + [os.path.join(CSRC, s) for s in SOURCES] + list(extra) + ["-lcusolver"])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    srcs = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(ROOT, "include", "jolt.h")]
    return all(os.path.getmtime(s) <= t for s in srcs)


def build(force: bool = False, verbose: bool = True) -> str:
    if not force and up_to_date():
        return LIB
    cmd = nvcc_cmd()
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    tmp = LIB + ".tmp"
    cmd[cmd.index("-o") + 1] = tmp
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv)
