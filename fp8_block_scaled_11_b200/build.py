"""Build step for the CUDA library: csrc/fp8bs_lib.cu -> libfp8bs.so (in-tree).

Compiled for sm_100a only (B200), no fast-math: the quantization's fp32
division and reciprocal must be IEEE round-to-nearest.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
MAIN = os.path.join(SRC_DIR, "fp8bs_lib.cu")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(HERE, "libfp8bs.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _sources():
    out = [os.path.join(INCLUDE, "fp8bs.h")]
    for f in sorted(os.listdir(SRC_DIR)):
        if f.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(SRC_DIR, f))
    return out


def needs_build() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB_PATH
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, "-I", INCLUDE, MAIN, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))
