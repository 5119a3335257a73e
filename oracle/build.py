"""Build the CPU oracle's shared library (test infrastructure).

Compiles ``nosa_oracle.c`` into ``libnosa_oracle.so`` next to it with gcc
(``-O2 -fopenmp``, no fast-math, so fp64 arithmetic keeps IEEE semantics).
Run ``python oracle/build.py`` or call :func:`build`.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "nosa_oracle.c")
LIB = os.path.join(HERE, "libnosa_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", SRC, "-o", LIB, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
