"""Compile the CPU oracle into oracle/liboracle.so (plain g++, C++17), and the
CPU baseline restated from the pages' binary_gemm_u64 into oracle/libk1.so.

Both are test and benchmark infrastructure: the tests, the smoke check and the
bench's CPU-baseline leg load them.  No floating-point contraction or
fast-math is allowed, so the compiled code keeps IEEE semantics operation by
operation.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bnn_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(
            os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "bnn_oracle.h"))):
        return LIB
    cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
           "-shared", "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


K1_SRC = os.path.join(HERE, "k1_popcount.cpp")
K1_LIB = os.path.join(HERE, "libk1.so")


def build_k1(force: bool = False) -> str:
    """The CPU baseline (row-by-row XOR + 64-bit popcount, OpenMP over rows)."""
    if not force and os.path.exists(K1_LIB) and os.path.getmtime(K1_LIB) >= os.path.getmtime(K1_SRC):
        return K1_LIB
    cmd = ["g++", "-std=c++20", "-O3", "-mpopcnt", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
           "-shared", "-Wall", "-Wextra", "-o", K1_LIB + ".tmp", K1_SRC]
    subprocess.run(cmd, check=True)
    os.replace(K1_LIB + ".tmp", K1_LIB)
    return K1_LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
    print(build_k1(force="--force" in sys.argv))
