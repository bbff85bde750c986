"""Compile the C oracle into ``oracle/libbsp_oracle.so`` (test infrastructure).

Plain C11, ``-O2 -ffp-contract=off`` and no fast-math, so each float expression in
the oracle is one correctly rounded IEEE binary32 operation.  OpenMP only splits
independent rows across host threads.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bsp_oracle.c")
LIB = os.path.join(HERE, "libbsp_oracle.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
