"""Build step of libvsa.so: one nvcc invocation, in-tree, for sm_100a.

    python -m block_sparse_attention_pool_b200.build [--force]

The library is a single translation unit (csrc/vsa.cu includes every kernel
header) compiled with cudart linked statically, so the shared object needs no
CUDA runtime at load time and only the driver when a call runs.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libvsa.so")
HEADER = os.path.join(ROOT, "include", "vsa.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xcompiler", "-fvisibility=hidden",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _sources():
    out = [HEADER]
    for name in sorted(os.listdir(SRC_DIR)):
        if name.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(SRC_DIR, name))
    return out


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in _sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [_nvcc(), *NVCC_FLAGS, "-o", LIB + ".tmp", os.path.join(SRC_DIR, "vsa.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
