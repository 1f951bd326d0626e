"""Compile the C oracle (test infrastructure) twice from the same source:
``oracle/libkvq_oracle.so``, single-threaded (the oracle the tests use), and
``oracle/libkvq_oracle_omp.so`` with OpenMP, whose outer loops over rows, keys or
(batch, head) units run on all host cores (the all-cores CPU baseline; every row, key or
unit is computed as in the single-threaded build).

Flags keep every fp32 operation a single IEEE-754 round-to-nearest-even operation:
no fast-math, no FMA contraction.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kvq_oracle.c")
LIB = os.path.join(HERE, "libkvq_oracle.so")
LIB_OMP = os.path.join(HERE, "libkvq_oracle_omp.so")
FLAGS = ["-O2", "-std=c11", "-D_GNU_SOURCE", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
         "-Wall", "-Wextra"]


def _build_one(lib: str, extra, force: bool) -> str:
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= os.path.getmtime(SRC):
        return lib
    subprocess.run(["gcc"] + FLAGS + extra + ["-o", lib, SRC, "-lm"], check=True)
    return lib


def build(force: bool = False, all_cores: bool = False) -> str:
    """Build both variants if stale; return the path of the one asked for."""
    plain = _build_one(LIB, ["-Wno-unknown-pragmas"], force)
    omp = _build_one(LIB_OMP, ["-fopenmp"], force)
    return omp if all_cores else plain


if __name__ == "__main__":
    print(build(force=True), build(all_cores=True))
