"""Compile the CPU oracle into oracle/liblores_oracle.so (test infrastructure).

Plain gcc, no fast-math, no fp contraction: the oracle's fp32 arithmetic must
be exactly the operations written in lores_oracle.c.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lores_oracle.c")
LIB = os.path.join(HERE, "liblores_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-frounding-math",
           "-fno-fast-math", "-fPIC", "-shared", "-o", LIB, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
