"""Build the CUDA libraries in-tree: rotated_w4a4_quantized_b200/libconvrot.so
(the W4A4 layer, include/convrot.h), libconvrot_w4a16.so (the W4A16
variant, include/convrot_w4a16.h) and libconvrot_nvfp4.so (the NVFP4
variant, include/convrot_nvfp4.h).

    python -m rotated_w4a4_quantized_b200.build [--verbose]

Each library is one translation unit (csrc/convrot.cu, csrc/w4a16.cu,
csrc/nvfp4.cu)
compiled for sm_100a only, with IEEE
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
_INC = os.path.join(os.path.dirname(HERE), "include")
SRC = os.path.join(HERE, "csrc", "convrot.cu")
DEPS = [os.path.join(HERE, "csrc", f) for f in ("convrot.cu", "gemm.cuh", "prep.cuh", "ptx.cuh",
                                                     "skinny.cuh", "decode.cuh")]
HEADER = os.path.join(_INC, "convrot.h")
LIB = os.path.join(HERE, "libconvrot.so")
SRC_W4A16 = os.path.join(HERE, "csrc", "w4a16.cu")
DEPS_W4A16 = [os.path.join(HERE, "csrc", f) for f in ("w4a16.cu", "prep.cuh", "ptx.cuh")] + [
    HEADER, os.path.join(_INC, "convrot_w4a16.h")]
LIB_W4A16 = os.path.join(HERE, "libconvrot_w4a16.so")
SRC_NVFP4 = os.path.join(HERE, "csrc", "nvfp4.cu")
DEPS_NVFP4 = [os.path.join(HERE, "csrc", f) for f in ("nvfp4.cu", "prep.cuh", "ptx.cuh")] + [
    HEADER, os.path.join(_INC, "convrot_nvfp4.h")]
LIB_NVFP4 = os.path.join(HERE, "libconvrot_nvfp4.so")

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


def _stale(lib: str, deps) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in deps)


def stale() -> bool:
    return (_stale(LIB, DEPS + [HEADER]) or _stale(LIB_W4A16, DEPS_W4A16)
            or _stale(LIB_NVFP4, DEPS_NVFP4))


def _build_one(src: str, lib: str, verbose: bool) -> None:
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, src, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False) -> str:
    """Build whichever library is missing or older than its sources; returns
    the W4A4 library's path."""
    if force or _stale(LIB, DEPS + [HEADER]):
        _build_one(SRC, LIB, verbose)
    if force or _stale(LIB_W4A16, DEPS_W4A16):
        _build_one(SRC_W4A16, LIB_W4A16, verbose)
    if force or _stale(LIB_NVFP4, DEPS_NVFP4):
        _build_one(SRC_NVFP4, LIB_NVFP4, verbose)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
    print(LIB_W4A16)
    print(LIB_NVFP4)
