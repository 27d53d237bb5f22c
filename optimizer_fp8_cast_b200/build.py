"""Build libfp8train.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a.

    python -m optimizer_fp8_cast_b200.build [--verbose-ptxas]

One translation unit (csrc/fp8train.cu) holds every kernel, so the device error word is a
single symbol. No fast-math: the quantise, scale and AdamW arithmetic relies on IEEE rounding.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
MAIN = os.path.join(SRC_DIR, "fp8train.cu")
HEADER = os.path.join(ROOT, "include", "fp8train.h")
LIB = os.path.join(HERE, "libfp8train.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _sources():
    out = [HEADER]
    for f in os.listdir(SRC_DIR):
        if f.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(SRC_DIR, f))
    return out


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
           "-o", tmp, MAIN]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv))
