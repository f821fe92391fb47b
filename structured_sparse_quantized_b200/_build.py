"""Build libss.so (the C-ABI CUDA library) in-tree for sm_100a.

    python -m structured_sparse_quantized_b200._build

nvcc compiles csrc/ss_api.cu (which includes every kernel) with
-gencode arch=compute_100a,code=sm_100a; the CUDA runtime is linked
statically, so the library loads on a machine without a GPU (every call
then returns an error) and needs only the driver on a GPU machine.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC_DIR = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libss.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "--expt-relaxed-constexpr"]


def _sources():
    files = [os.path.join(SRC_DIR, f) for f in os.listdir(SRC_DIR)]
    files.append(os.path.join(ROOT, "include", "ss.h"))
    return files


def build(force: bool = False, verbose: bool = False) -> str:
    newest = max(os.path.getmtime(f) for f in _sources())
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    cmd = [NVCC, *FLAGS, "-I", os.path.join(ROOT, "include"), "-I", SRC_DIR,
           "-o", LIB, os.path.join(SRC_DIR, "ss_api.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
