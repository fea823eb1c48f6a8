"""Build the CPU oracle (test infrastructure) into oracle/liboracle.so with plain gcc.

Flags: -O2 without -ffast-math, and -ffp-contract=off so that no multiply-add is fused:
the oracle's fp32 steps are each a single correctly rounded operation.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "sq_oracle.c")
HDR = os.path.join(HERE, "sq_oracle.h")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-std=gnu11", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wextra", "-Wno-unused-parameter"]


def build(force: bool = False) -> str:
    """Compile liboracle.so if it is missing or older than its sources; return its path."""
    newest = max(os.path.getmtime(SRC), os.path.getmtime(HDR), os.path.getmtime(__file__))
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
