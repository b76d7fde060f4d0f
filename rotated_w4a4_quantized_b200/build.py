"""Build the CUDA library in-tree: rotated_w4a4_quantized_b200/libconvrot.so.

    python -m rotated_w4a4_quantized_b200.build [--verbose]

Compiles csrc/convrot.cu (one translation unit) for sm_100a only, with IEEE
fp32 semantics (no fast-math: the epilogue and the quantiser rely on
correctly rounded multiply, add and divide).  The CUDA runtime is linked
statically; the driver's tensor-map encoder is looked up at run time, so no
link against libcuda is needed and the build runs on a machine without a GPU.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "convrot.cu")
DEPS = [os.path.join(HERE, "csrc", f) for f in ("convrot.cu", "gemm.cuh", "prep.cuh", "ptx.cuh",
                                                     "skinny.cuh", "decode.cuh")]
HEADER = os.path.join(os.path.dirname(HERE), "include", "convrot.h")
LIB = os.path.join(HERE, "libconvrot.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in DEPS + [HEADER])


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, SRC, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
