"""Build the in-tree CUDA library ``libonebit.so`` for sm_100a with nvcc.

``python bit_adam_error_b200/build.py`` (run as a file: importing the package
loads the library this script builds) or ``build()`` compiles
``csrc/onebit.cu`` into ``bit_adam_error_b200/libonebit.so``.  The library is
self-contained (static CUDA runtime) and exports the C ABI of
``include/onebit.h``.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libonebit.so")
SOURCES = [os.path.join(CSRC, "onebit.cu")]
DEPS = SOURCES + [os.path.join(CSRC, "kernels.cuh"), os.path.join(CSRC, "ternary.cuh"),
                  os.path.join(CSRC, "twobit.cuh"), os.path.join(INCLUDE, "onebit.h")]

# -fmad=false: no FMA contraction, so every fp32 expression rounds as written;
# IEEE division and square root; no fast-math.
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-fmad=false", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
    "-Xcompiler", "-fPIC,-O2", "-shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libonebit.so")


def _stale(out: str, deps) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile libonebit.so if it is missing or older than its sources."""
    if not force and not _stale(LIB, DEPS):
        return LIB
    cmd = [nvcc(), *NVCC_FLAGS, *extra, f"-I{INCLUDE}", f"-I{CSRC}", "-o", LIB + ".tmp", *SOURCES]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    v = "-v" in sys.argv
    print(build(force="--force" in sys.argv, verbose=v,
                extra=("-Xptxas", "-v") if "--ptxas-v" in sys.argv else ()))
