"""Build the fp64 CPU oracle (test infrastructure; never part of the product path).

``python -m oracle.build`` compiles ``unstep_oracle.c`` into ``liboracle.so`` next to this file
with gcc and OpenMP.  No fast-math: the oracle relies on IEEE double semantics.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "unstep_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def needs_build() -> bool:
    return (not os.path.exists(LIB)) or os.path.getmtime(LIB) < os.path.getmtime(SRC)


def build(force: bool = False) -> str:
    if force or needs_build():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-shared",
               "-fPIC", "-std=c11", "-Wall", "-o", tmp, SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
