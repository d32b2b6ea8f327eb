"""Build the CUDA library libcr_w4a8.so in-tree for sm_100a.

    python -m w4a8_codebook_quantized_b200.build [--force] [--verbose]

One nvcc invocation over csrc/cr_lib.cu (the kernels are header files of that
translation unit), static CUDA runtime, no fast-math: the kernels rely on
IEEE division, round-to-nearest conversions and unfused fp32 operations
where the layer's arithmetic is defined that way.
"""
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libcr_w4a8.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-I", INCLUDE, "-I", CSRC,
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def nvcc() -> str:
    cand = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    p = os.path.join(cand, "bin", "nvcc")
    return p if os.path.exists(p) else "nvcc"


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libcr_w4a8.so if it is missing or older than any source."""
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(s) for s in _sources())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, os.path.join(CSRC, "cr_lib.cu"), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
