"""Compile the C oracle (test infrastructure) into oracle/liboracle.so with gcc.

Plain -O2 without -ffast-math, so the compiler may not reassociate floating point.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "titans_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False, src: str = SRC, out: str = LIB, extra=()) -> str:
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-Wall", "-Wextra",
           *extra, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
