"""Build the CPU oracle's shared library (test infrastructure only).

``python -m oracle.build`` (or ``build()``) compiles ``jl_oracle.c`` with gcc
and OpenMP into ``oracle/libjl_oracle.so``.  Building the checker is not using
it: the product library never links or loads this file.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "jl_oracle.c")
LIB = os.path.join(HERE, "libjl_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(
        os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "jl_oracle.h"))
    ):
        return LIB
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", LIB, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
