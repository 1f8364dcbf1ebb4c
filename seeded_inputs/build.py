"""Build the seeded-input generator libraries in place.

libseeded_inputs.so       host fill (gcc, OpenMP)
libseeded_inputs_cuda.so  device fill (nvcc, sm_100a)
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(HERE, "libseeded_inputs.so")
CUDA_LIB = os.path.join(HERE, "libseeded_inputs_cuda.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def _run(cmd):
    subprocess.run(cmd, check=True, cwd=HERE)


def build(force=False, cuda=True):
    hdr = os.path.join(HERE, "philox.h")
    host_src = os.path.join(HERE, "gen_host.c")
    if force or _stale(HOST_LIB, [host_src, hdr]):
        _run(["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared",
              "-ffp-contract=off", "-Wall", "-o", HOST_LIB, host_src])
    cuda_src = os.path.join(HERE, "gen_cuda.cu")
    if cuda and (force or _stale(CUDA_LIB, [cuda_src, hdr])):
        _run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
              "-fmad=false", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
              "-o", CUDA_LIB, cuda_src])


if __name__ == "__main__":
    build(force=True)
