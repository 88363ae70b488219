"""Compile the plain-C oracle into ``oracle/libgq_oracle.so``.

Test infrastructure only: the oracle is built so that tests, the smoke check
and the benchmark's CPU-baseline leg can run it.  Building the checker is not
using it; the product library never links or loads this file.

Flags: ``-O2 -ffp-contract=off`` (no fused multiply-add contraction),
``-fno-fast-math`` and SSE binary32 arithmetic (x86-64 default), so every
floating-point operation in the oracle is one correctly rounded IEEE op.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gq_oracle.c")
LIB = os.path.join(HERE, "libgq_oracle.so")

CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
          "-fno-builtin-nearbyintf", "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle if the library is missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
