"""Build the oracle's shared library (plain C, host only).

TEST INFRASTRUCTURE: the oracle is loaded only by the test suite, the smoke
check and the benchmark's CPU-baseline leg.

Flags: -ffp-contract=off keeps every a*b+c as a separate multiply and add;
no fast-math, so division and sqrtf are the correctly rounded IEEE operations
and subnormals are kept.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "zero_ref.c")
HDR = os.path.join(HERE, "zero_ref.h")
LIB = os.path.join(HERE, "libzero_ref.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-fexcess-precision=standard", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    newest = max(os.path.getmtime(SRC), os.path.getmtime(HDR), os.path.getmtime(__file__))
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
