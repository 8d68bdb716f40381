"""Builds libhaste.so (sm_100a) in-tree with nvcc.

The library is one translation unit (api.cu includes the kernel sources), linked
against the static CUDA runtime so that it depends only on the driver.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
OUT = os.path.join(PKG, "libhaste.so")
def _sources():
    """Every CUDA source and header of the library, and the ABI header."""
    own = [f for f in os.listdir(HERE) if f.endswith((".cu", ".cuh"))]
    return own + [os.path.join("..", "..", "include", "haste.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "--expt-relaxed-constexpr", "-maxrregcount=152", "-Xcompiler", "-fPIC,-O2", "-shared"]


def stale() -> bool:
    if not os.path.exists(OUT):
        return True
    t = os.path.getmtime(OUT)
    return any(os.path.getmtime(os.path.join(HERE, s)) > t for s in _sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if force or stale():
        tmp = OUT + f".tmp{os.getpid()}"
        cmd = [NVCC, *FLAGS, *(["-Xptxas", "-v"] if verbose else []), "-o", tmp,
               os.path.join(HERE, "api.cu")]
        subprocess.check_call(cmd, cwd=HERE)
        os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(OUT)
