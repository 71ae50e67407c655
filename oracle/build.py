"""Builds the CPU oracle (``oracle/liboracle.so``) with gcc.

The oracle is test infrastructure: only the tests, the package smoke check and
the benchmark's CPU-baseline leg load it.  Built with -O2, no fast-math and no
floating-point contraction (so the double arithmetic is the plain IEEE
arithmetic the formulas ask for, one rounding per operation), with OpenMP so
loops over independent tokens/rows may use several host cores; the per-row
arithmetic does not depend on the thread count.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", "-Wall", "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
