"""Build the lbq CUDA library (liblbq.so) in-tree for sm_100a.

Run ``python bit_weight_only_pack_b200/build.py`` (or call :func:`build`); this
script does not import the package, so it works while the library is stale.
The library is one translation unit (csrc/lbq.cu includes every kernel).
"""

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "liblbq.so")
SOURCES = [os.path.join(PKG, "csrc", "lbq.cu")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(verbose=False, extra=()):
    """Compile liblbq.so (static cudart, -O3, -lineinfo) and return its path."""
    deps = SOURCES + [os.path.join(PKG, "csrc", f) for f in os.listdir(os.path.join(PKG, "csrc"))]
    deps.append(os.path.join(ROOT, "include", "lbq.h"))
    if os.path.exists(LIB) and not extra:
        newest = max(os.path.getmtime(d) for d in deps)
        if os.path.getmtime(LIB) >= newest:
            return LIB
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
           "-cudart", "static", "-I", os.path.join(ROOT, "include"), "-o", LIB + ".tmp", *SOURCES, *extra]
    if verbose:
        cmd.append("-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
