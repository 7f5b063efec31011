"""Build the CPU oracle (oracle/libkvqref.so) with g++.

Test infrastructure: the oracle is compiled here so that the tests, the smoke
check and the benchmark's CPU-baseline leg can load it.  Nothing in the CUDA
library links against it.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCES = [os.path.join(HERE, "kvqref.cpp")]
HEADERS = [os.path.join(HERE, "kvqref.h")]
LIB = os.path.join(HERE, "libkvqref.so")

# IEEE binary32 arithmetic with no contraction and no fast-math rewrites.
CXXFLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off",
            "-fno-fast-math", "-fexcess-precision=standard", "-Wall", "-Wextra"]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS + [__file__])


def build(force: bool = False) -> str:
    if force or _stale():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["g++", *CXXFLAGS, *SOURCES, "-o", tmp]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
