"""Compile the CPU oracle (``rece_oracle.c``) into ``oracle/librece_oracle.so``.

Test infrastructure: the oracle is built so that the tests, the smoke check and the
benchmark's CPU-baseline leg can call it.  Plain gcc, OpenMP over rows, no fast-math
and no floating-point contraction (every fused multiply-add is an explicit ``fmaf``).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "rece_oracle.c")
LIB = os.path.join(HERE, "librece_oracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Build the shared library if it is missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
