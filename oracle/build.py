"""Build the CPU oracle (plain C) into oracle/_build/liboracle.so with gcc.

Test infrastructure only: the product library never links or loads it.
Flags: -O2 without fast-math and with -ffp-contract=off so that each fp64
operation in the oracle is the IEEE operation written in the source.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csa2_oracle.c")
HDR = os.path.join(HERE, "csa2_oracle.h")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "liboracle.so")
LIB_OMP = os.path.join(OUT_DIR, "liboracle_omp.so")     # same source, OpenMP on (host-core timing only)


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in (SRC, HDR, __file__))


def build(force: bool = False, openmp: bool = False) -> str:
    """Build the test oracle (single-threaded), or with openmp=True the same
    source with its "omp parallel for" loops active."""
    lib = LIB_OMP if openmp else LIB
    if force or needs_build(lib):
        os.makedirs(OUT_DIR, exist_ok=True)
        tmp = lib + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c99", "-O2", "-fPIC", "-shared",
               "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra"]
        cmd += ["-fopenmp"] if openmp else ["-Wno-unknown-pragmas"]
        cmd += ["-o", tmp, SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
    print(build(force="--force" in sys.argv, openmp=True))
