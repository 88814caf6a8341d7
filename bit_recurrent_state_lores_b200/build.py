"""Build liblores.so (the C-ABI library) in-tree for sm_100a with nvcc.

    python -m bit_recurrent_state_lores_b200.build [--verbose]

No fast-math: the kernels' fp32 rounding is part of the state format, so every
rounding-sensitive operation is written with explicit round-to-nearest intrinsics
and fma contraction is disabled as a second guard.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "lores.cu")
DEPS = [SRC, os.path.join(PKG, "csrc", "lores_device.cuh"), os.path.join(ROOT, "include", "lores.h")]
LIB = os.path.join(PKG, "liblores.so")
NVCC = os.environ.get("NVCC", "nvcc")


SRCS = [SRC, os.path.join(PKG, "csrc", "lores_mt.cu")]
DEPS += SRCS[1:] + [os.path.join(PKG, "csrc", "lores_step.cuh")]
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-fmad=false", "-Xcompiler", "-fPIC"]


def nvcc_cmd(out=LIB, verbose=False):
    """One-shot command line (both translation units in one nvcc call)."""
    cmd = [NVCC] + FLAGS + ["-shared", "-I", os.path.join(ROOT, "include"), "-o", out] + SRCS
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the translation units in parallel, then link the shared library."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(p) for p in DEPS)):
        return LIB
    objs, procs = [], []
    for src in SRCS:
        obj = os.path.join(PKG, "csrc", os.path.basename(src)[:-3] + ".o")
        cmd = [NVCC] + FLAGS + (["-Xptxas=-v"] if verbose else []) + [
            "-I", os.path.join(ROOT, "include"), "-c", "-o", obj, src]
        procs.append(subprocess.Popen(cmd))
        objs.append(obj)
    codes = [pr.wait() for pr in procs]
    if any(codes):
        raise subprocess.CalledProcessError(max(codes), "nvcc")
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", LIB]
                   + objs, check=True)
    for obj in objs:
        os.remove(obj)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
