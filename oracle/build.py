"""Build the float64 oracle (oracle.c) into oracle/liboracle.so with gcc + OpenMP.

Test infrastructure: the product library never links or loads this file.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(src: str = SRC, out: str = LIB, extra=()) -> str:
    """Compile ``src`` into the shared library ``out`` (rebuilt when stale)."""
    if (os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src)
            and not extra):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-Wno-unused-parameter", *extra, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(*sys.argv[1:2]))
