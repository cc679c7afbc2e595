"""Compile the CPU oracle (oracle.c) into oracle/liboracle.so.

Test infrastructure: the library is used by the test-suite, the smoke check
and the CPU-baseline leg of the benchmark only.  Floating-point contraction
and fast-math are off so each float operation in oracle.c is one IEEE-754
binary32 operation rounded to nearest even.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = [
    "-O2",
    "-std=c11",
    "-ffp-contract=off",
    "-fno-fast-math",
    "-fno-finite-math-only",
    "-fopenmp",
    "-fPIC",
    "-shared",
    "-Wall",
    "-Wextra",
    "-Wno-unused-parameter",
]


def build(force: bool = False) -> str:
    """Build liboracle.so if it is missing or older than oracle.c; return its path."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc"] + CFLAGS + [SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
