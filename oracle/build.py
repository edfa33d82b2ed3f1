"""Compile the CPU oracle (plain single-threaded C++) into oracle/libmlxq_oracle.so.

Test infrastructure: the library built here is the independent checker of the
CUDA path and is loaded only by the tests, the smoke check and the benchmark's
CPU-baseline leg.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mlxq_oracle.cpp")
LIB = os.path.join(HERE, "libmlxq_oracle.so")

# -ffp-contract=off: no silent fusing of a*b+c; the source writes std::fma
# where the definition has one.  -fno-fast-math keeps IEEE semantics.
CXXFLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["g++", *CXXFLAGS, SRC, "-o", LIB + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
