"""Build the oracle's C library in place (gcc, single-threaded, no FMA contraction)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "liboracle.so")
SRC = os.path.join(HERE, "oracle.c")


def build(force=False):
    if force or not os.path.exists(LIB) or os.path.getmtime(SRC) > os.path.getmtime(LIB):
        subprocess.run(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
                        "-fPIC", "-shared", "-Wall", "-o", LIB, SRC, "-lm"],
                       check=True, cwd=HERE)


if __name__ == "__main__":
    build(force=True)
