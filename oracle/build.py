"""Build the fp64 CPU oracle (``liboracle.so``) with the host C compiler.

Test infrastructure: see ``gn_oracle.h``. Run as ``python -m oracle.build`` or through
``oracle.build.build()``; the result lands next to this file.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gn_oracle.c")
HDR = os.path.join(HERE, "gn_oracle.h")
LIB = os.path.join(HERE, "liboracle.so")


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in (SRC, HDR, __file__))


def build(force: bool = False) -> str:
    """Compile the oracle if its sources are newer than the library; return the library path."""
    if force or stale():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [os.environ.get("CC", "gcc"), "-std=c11", "-D_DEFAULT_SOURCE", "-O2",
               "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", "-Wall", "-Wextra",
               "-o", tmp, SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
