"""Compile the float64 oracle (plain C) into oracle/libeqlin_oracle.so.

TEST INFRASTRUCTURE ONLY: the oracle is what the CUDA path is checked
against.  Building it is not using it; only the tests, the package smoke
check and bench.py's CPU-baseline leg load the result.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "eqlin_oracle.c")
LIB = os.path.join(HERE, "libeqlin_oracle.so")


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the oracle if the .so is missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-o", tmp, SRC, "-lm"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
