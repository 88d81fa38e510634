"""Build the CPU oracle (test infrastructure) into oracle/liboracle.so.

Plain C, IEEE fp32/fp64 with no FMA contraction and no fast-math, so every fp32
operation in the oracle is one round-to-nearest-even step. Called by the test
suite, by __graft_entry__.build() and by bench.py's CPU-baseline leg.

liboracle_omp.so is the same source with -fopenmp (row loops spread over the host
cores, each row computed by the same code); only bench.py's oracle timing uses it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "macaq_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
LIB_OMP = os.path.join(HERE, "liboracle_omp.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-fexcess-precision=standard", "-Wall", "-Wextra"]


def _build(lib, extra, force):
    deps = [SRC, os.path.join(HERE, "macaq_oracle.h"), os.path.abspath(__file__)]
    if not force and os.path.exists(lib):
        lib_t = os.path.getmtime(lib)
        if all(os.path.getmtime(d) <= lib_t for d in deps):
            return lib
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, *extra, "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False) -> str:
    """The single-threaded oracle (the OpenMP pragmas are ignored)."""
    return _build(LIB, ["-Wno-unknown-pragmas"], force)


def build_omp(force: bool = False) -> str:
    """The same oracle with its row loops on all host cores (OpenMP)."""
    return _build(LIB_OMP, ["-fopenmp"], force)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
    print(build_omp(force="--force" in sys.argv))
