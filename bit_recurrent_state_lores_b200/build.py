"""Build liblores.so (the C-ABI library) in-tree for sm_100a with nvcc.

    python -m bit_recurrent_state_lores_b200.build [--verbose] [--checked]

csrc/lores.cu (host side, loader, dequantizer) and 45 compilations of csrc/lores_inst.cu
(one decode-step kernel family per key width x single/multi-token x storage family --
plain; dense and per-lane; per-lane only --, one two-rows-per-lane family per key width x
single/multi-token, and one key-axis family per key width) build in parallel, one nvcc
process per CPU core, then link.

--checked builds liblores_checked.so instead: the same sources compiled with
LORES_INDEX_CHECKS, so that every global access of the kernels is checked against the
extent of its buffer first (include/lores.h, lores_index_checked); a debugging build, not
the product.

No fast-math: the kernels' fp32 rounding is part of the state format, so every
rounding-sensitive operation is written with explicit round-to-nearest intrinsics
and fma contraction is disabled as a second guard.
"""
import os
import subprocess
import sys
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
SRC = os.path.join(CSRC, "lores.cu")
INST = os.path.join(CSRC, "lores_inst.cu")
DEPS = [SRC, INST, os.path.join(CSRC, "lores_step.cuh"), os.path.join(CSRC, "lores_device.cuh"),
        os.path.join(CSRC, "lores_key.cuh"), os.path.join(CSRC, "lores_pair.cuh"),
        os.path.join(CSRC, "lores_mma.cuh"),
        os.path.join(ROOT, "include", "lores.h")]
LIB = os.path.join(PKG, "liblores.so")
LIB_CHECKED = os.path.join(PKG, "liblores_checked.so")
NVCC = os.environ.get("NVCC", "nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-fmad=false", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include")]
KEY_WIDTHS = (16, 32, 64, 128, 256)
MMA_WIDTHS = (16, 32, 64, 128)       # key widths of the tensor-core kernel


def units():
    """(source, extra flags, object name) of every compilation, the slowest first (the
    extended families), so the parallel build does not end on one long unit."""
    out = []
    for ext in (1, 4, 3, 2, 0):
        for mt in (1, 0):
            for dk in reversed(KEY_WIDTHS):
                out.append((INST, [f"-DLORES_DK={dk}", f"-DLORES_MT={mt}", f"-DLORES_EXT={ext}"],
                            f"lores_inst_{dk}_{mt}_{ext}.o"))
    for mt in (1, 0):
        for dk in reversed(KEY_WIDTHS):
            out.append((INST, [f"-DLORES_DK={dk}", "-DLORES_PAIR=1", f"-DLORES_MT={mt}"],
                        f"lores_pair_{dk}_{mt}.o"))
    for dk in MMA_WIDTHS:
        out.append((INST, [f"-DLORES_DK={dk}", "-DLORES_MMA=1"], f"lores_mma_{dk}.o"))
    for dk in KEY_WIDTHS:
        out.append((INST, [f"-DLORES_DK={dk}", "-DLORES_KEY=1"], f"lores_key_{dk}.o"))
    out.append((SRC, [], "lores.o"))
    return out


def build(force: bool = False, verbose: bool = False, jobs: int = 0,
          checked: bool = False) -> str:
    """Compile every unit (up to `jobs` at a time, default: the CPU count), then link.
    checked: the index-checked library instead of the product."""
    lib = LIB_CHECKED if checked else LIB
    mode = ["-DLORES_INDEX_CHECKS=1"] if checked else []
    if (not force and os.path.exists(lib)
            and os.path.getmtime(lib) >= max(os.path.getmtime(p) for p in DEPS)):
        return lib
    jobs = jobs or max(1, os.cpu_count() or 1)
    with tempfile.TemporaryDirectory(prefix="lores_build_") as tmp:
        pending = list(units())
        running, objs = [], []
        while pending or running:
            while pending and len(running) < jobs:
                src, extra, name = pending.pop(0)
                obj = os.path.join(tmp, name)
                cmd = [NVCC] + FLAGS + mode + extra + (["-Xptxas=-v"] if verbose else []) + [
                    "-c", "-o", obj, src]
                running.append((subprocess.Popen(cmd), name))
                objs.append(obj)
            proc, name = running.pop(0)
            if proc.wait() != 0:
                for p, _ in running:
                    p.wait()
                raise subprocess.CalledProcessError(proc.returncode, f"nvcc ({name})")
        subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o",
                        lib + ".tmp"] + objs, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv, checked="--checked" in sys.argv))
