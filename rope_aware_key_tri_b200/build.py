"""Build the sm_100a CUDA library (``lib/libtri_b200.so``) with nvcc.

The library is compiled in-tree so it travels with the source tree; nothing is
installed into site-packages and there is no JIT step at import time.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIBDIR = os.path.join(HERE, "lib")
LIB = os.path.join(LIBDIR, "libtri_b200.so")
SOURCES = [os.path.join(CSRC, "tri_api.cu")]
EXPORTS = os.path.join(CSRC, "exports.map")
DEPS = SOURCES + [os.path.join(CSRC, "tri_kernel.cuh"), os.path.join(CSRC, "tri_calib.cuh"), os.path.join(CSRC, "tri_append.cuh"), os.path.join(CSRC, "tri_maxdelta.cuh"), os.path.join(CSRC, "tri_attend.cuh"), os.path.join(ROOT, "include", "tri.h"), EXPORTS]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    os.makedirs(LIBDIR, exist_ok=True)
    cmd = [nvcc()] + NVCC_FLAGS + (["-Xptxas", "-v"] if verbose else []) + \
        ["-Xlinker", "--version-script=" + EXPORTS, "-I", os.path.join(ROOT, "include"), "-o", LIB] + SOURCES
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
