"""Build liblb.so (the C-ABI library) in-tree for sm_100a with nvcc.

python -m moe_expert_load_bf16_b200.build [--force] [--debug]
"""
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblb.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  [os.path.join(INCLUDE, "lb.h")])


def build(force: bool = False, verbose: bool = False, extra=(), out: str = LIB) -> str:
    """Compile lb.cu into `out` (the product library by default) unless it is
    newer than every source.  `extra` adds nvcc flags (e.g. -DLB_TIMING for
    the phase-timing build, which goes to its own file)."""
    newest = max(os.path.getmtime(s) for s in sources())
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC,
           os.path.join(CSRC, "lb.cu"), "-o", out]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    extra = ["-Xptxas", "-v"] if "--ptxas" in sys.argv else []
    print(build(force="--force" in sys.argv, verbose=True, extra=extra))
