"""Build libi8linear.so in-tree for sm_100a with nvcc (no GPU needed to compile).

    python -m bit_matmul_decomposition_b200.build [--verbose]

The library is one translation unit (csrc/api.cu includes every kernel), linked against
the static CUDA runtime, so it loads on a machine without a GPU driver; the driver's
tensor-map encoder is looked up at run time.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libi8linear.so")
SOURCES = ["api.cu", "common.cuh", "quant.cuh", "gemm.cuh", "gemm_wide.cuh", "gemv.cuh", "bwd.cuh"]
HEADER = os.path.join(ROOT, "include", "i8linear.h")

NVCC_FLAGS = [
    "-std=c++17", "-O3", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
]


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES] + [HEADER]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + ".%d.tmp" % os.getpid()
    cmd = [_nvcc()] + NVCC_FLAGS + (["-Xptxas", "-v"] if verbose else []) + [
        "-I", os.path.join(ROOT, "include"), os.path.join(CSRC, "api.cu"), "-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
