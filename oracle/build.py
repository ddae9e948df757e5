"""Compile the fp64 CPU oracle (``lard_oracle.c``) into ``liblard_oracle.so``.

Test infrastructure only: the product path never loads the result.
Plain gcc, ``-O2`` without fast-math so that every double operation keeps
IEEE semantics, OpenMP for parallelism over independent rows/columns.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lard_oracle.c")
LIB = os.path.join(HERE, "liblard_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
           "-std=c11", "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
