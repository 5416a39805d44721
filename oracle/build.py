"""Compile the fp64 oracle (test infrastructure) into oracle/libfboracle.so.

Plain gcc, -O2, no -march and no fast-math, so that IEEE fp64 semantics hold and
the library runs on any x86-64 host it is copied to.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fb_oracle.c")
LIB = os.path.join(HERE, "libfboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
           "-o", LIB, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
