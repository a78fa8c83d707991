"""Build the LoopKV CUDA library in-tree: libloopkv.so next to this file.

nvcc compiles every source under csrc/ for sm_100a only (no PTX for other
targets) and links the CUDA runtime statically, so the library loads in any
process that already holds a CUDA context (PyTorch's included).
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libloopkv.so")
SOURCES = ["loopkv_api.cu", "append.cu", "decode.cu", "planner.cpp", "selftest.cu"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-cudart", "static",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "loopkv.h"), __file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libloopkv.so if any source is newer than it; return its path."""
    if not force and not _stale():
        return LIB
    objs = []
    build_dir = os.path.join(HERE, "_build")
    os.makedirs(build_dir, exist_ok=True)
    for src in SOURCES:
        obj = os.path.join(build_dir, os.path.splitext(src)[0] + ".o")
        cmd = [_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-Xptxas", "-v" if verbose else "-O3",
               "-c", os.path.join(CSRC, src), "-o", obj]
        subprocess.run(cmd, check=True, stdout=None if verbose else subprocess.DEVNULL,
                       stderr=None if verbose else subprocess.PIPE)
        objs.append(obj)
    tmp = LIB + ".tmp"
    subprocess.run([_nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-cudart", "static", *objs, "-o", tmp], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
