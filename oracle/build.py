"""Compile the CPU oracle (test and benchmark infrastructure).

    oracle/liblores_oracle.so       lores_oracle.c, single-threaded
    oracle/liblores_oracle_omp.so   lores_oracle.c + lores_oracle_omp.c with OpenMP: the
                                    same step over many tiles on all host cores

Plain gcc, no fast-math, no fp contraction: the oracle's fp32 arithmetic must
be exactly the operations written in lores_oracle.c.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lores_oracle.c")
SRC_OMP = os.path.join(HERE, "lores_oracle_omp.c")
LIB = os.path.join(HERE, "liblores_oracle.so")
LIB_OMP = os.path.join(HERE, "liblores_oracle_omp.so")
FLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-frounding-math", "-fno-fast-math", "-fPIC",
         "-shared"]


def _stale(lib, srcs):
    return not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(s) for s in srcs)


def build(force: bool = False) -> str:
    if force or _stale(LIB, [SRC]):
        subprocess.run(["gcc"] + FLAGS + ["-o", LIB, SRC, "-lm"], check=True)
    return LIB


def build_omp(force: bool = False) -> str:
    if force or _stale(LIB_OMP, [SRC, SRC_OMP]):
        subprocess.run(["gcc"] + FLAGS + ["-fopenmp", "-o", LIB_OMP, SRC, SRC_OMP, "-lm"],
                       check=True)
    return LIB_OMP


if __name__ == "__main__":
    print(build(force=True))
    print(build_omp(force=True))
