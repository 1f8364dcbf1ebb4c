"""Build libzero_b200.so in place: nvcc for sm_100a, IEEE-exact float flags.

-fmad=false keeps every multiply and add separately rounded (the kernels also use the
explicit __fadd_rn/__fmul_rn intrinsics); -prec-div / -prec-sqrt / -ftz=false keep
division and square root correctly rounded and subnormals intact.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libzero_b200.so")
# the same sources with ZERO_DEBUG: every located segment and tile is bounds-checked in the
# kernels (a failed check skips the tile and records ZERO_ERR_BOUNDS; nothing traps)
LIB_DEBUG = os.path.join(HERE, "libzero_b200_debug.so")
BUILD_DIR = os.path.join(ROOT, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SOURCES = ["layout.cpp", "kernels.cu", "bulk_step.cu", "abi.cu", "noalloc.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-fmad=false", "-prec-div=true", "-prec-sqrt=true",
         "-ftz=false", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "zero.h"))
    files.append(os.path.abspath(__file__))
    return files


def build(force=False, verbose_ptxas=False, debug=False):
    lib = LIB_DEBUG if debug else LIB
    if not force and os.path.exists(lib):
        t = os.path.getmtime(lib)
        if all(os.path.getmtime(f) <= t for f in _deps()):
            return lib
    out_dir = os.path.join(BUILD_DIR, "debug" if debug else "release")
    os.makedirs(out_dir, exist_ok=True)
    objs = []
    for src in SOURCES:
        obj = os.path.join(out_dir, src + ".o")
        extra = ["-Xptxas", "-v"] if verbose_ptxas and src.endswith(".cu") else []
        if debug:
            extra.append("-DZERO_DEBUG")
        subprocess.run([NVCC, *ARCH, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj], check=True)
        objs.append(obj)
    tmp = lib + ".tmp"
    subprocess.run([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-ldl"], check=True)
    os.replace(tmp, lib)
    return lib


def build_all(force=False):
    """The release library and its bounds-checking debug twin."""
    return build(force=force), build(force=force, debug=True)


if __name__ == "__main__":
    build(force=True, verbose_ptxas="-v" in sys.argv, debug="--debug" in sys.argv)
