"""Build the CPU oracle shared library (test infrastructure only).

    python oracle/build.py

Compiles ssref.c with gcc into oracle/libssref.so.  No fast-math and no
floating-point contraction, so every binary32 operation is one IEEE-rounded
operation as the oracle's comments state.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ssref.c")
LIB = os.path.join(HERE, "libssref.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra",
           "-o", LIB, SRC, "-lm"]
    subprocess.check_call(cmd)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
