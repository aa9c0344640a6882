"""Build libgdr.so (the CUDA library) in-tree for sm_100a with nvcc.

    python -m recurrent_state_memory_b200.build [--force]
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libgdr.so")
LIB_DEBUG = os.path.join(PKG, "libgdr_debug.so")    # every kernel's computed indices checked
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SOURCES = ["gdr.cu"]


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "gdr.h"))
    files.append(os.path.abspath(__file__))
    return files


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Build libgdr.so, or with debug=True libgdr_debug.so (-DGDR_BOUNDS_CHECK: every kernel
    tests the indices of the global-memory accesses it computes and reports a failure through
    the status word instead of making the access)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and os.path.exists(lib):
        newest = max(os.path.getmtime(f) for f in _deps())
        if os.path.getmtime(lib) >= newest:
            return lib
    tmp = lib + ".tmp"
    cmd = [NVCC, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC,
           "-o", tmp] + [os.path.join(CSRC, s) for s in SOURCES]
    if debug:
        cmd.insert(1, "-DGDR_BOUNDS_CHECK")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
