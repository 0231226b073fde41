"""Build the plain-C loop oracle (test infrastructure only) with gcc.

``python oracle/build_oracle.py`` writes ``oracle/_build/libmoe_oracle_loops.so``.
Building the checker does not use it; only the tests load the result.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_loops.c")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "libmoe_oracle_loops.so")


def build(force: bool = False) -> str:
    """Compile ``moe_loops.c`` into a shared library and return its path."""
    os.makedirs(OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + ".tmp"
    subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math", SRC,
                    "-o", tmp, "-lm"], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
