"""Compile the fp64 CPU oracle (plain C, gcc, OpenMP) into oracle/libtri_oracle.so.

Test infrastructure: building the checker is not using it. Only the tests,
the smoke check and the benchmark's CPU-baseline leg load the result.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "tri_oracle.c")
LIB = os.path.join(HERE, "libtri_oracle.so")


def build(force: bool = False, src: str = SRC, lib: str = LIB) -> str:
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= os.path.getmtime(src):
        return lib
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-Wall", "-Wextra",
           "-o", lib, src, "-lm"]
    subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
