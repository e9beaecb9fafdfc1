"""Compile the float64 CPU oracle (swa_oracle.c) into oracle/_swa_oracle.so with gcc.

Test infrastructure only: the oracle checks the CUDA library and is never part of it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "swa_oracle.c")
LIB = os.path.join(HERE, "_swa_oracle.so")


def build(src=SRC, out=LIB, extra=(), force=False):
    """Build the oracle shared library (OpenMP, -O2, no fast-math). Returns the path."""
    if (not force and os.path.exists(out) and src == SRC
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC",
           "-shared", "-std=c11", *extra, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
