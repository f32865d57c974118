"""Compile the oracle's C source into ``oracle/libmoc_oracle.so`` (gcc, OpenMP).

Building the checker is not using it: the package build step calls this so
that the tests and the CPU-baseline leg of the benchmark find the library.
No fast-math flags: the oracle's sums stay in the order the source states.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moc_oracle.c")
LIB = os.path.join(HERE, "libmoc_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
