"""Build the in-tree shared library ``libtg_gemm.so`` for sm_100a with nvcc.

Run ``python -m tiled_dense_gemm_fp16_b200.build`` (or call ``build()``).
The library is built in the package directory so that it travels with the
source tree; cudart is linked statically and the driver's tensor-map encoder
is looked up at run time, so the library needs no other CUDA library at load.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB_PATH = os.path.join(HERE, "libtg_gemm.so")
SOURCES = [os.path.join(CSRC, "tg_gemm.cu")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared",
              f"-I{os.path.join(ROOT, 'include')}"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libtg_gemm.so")


def _deps():
    deps = list(SOURCES)
    for name in os.listdir(CSRC):
        if name.endswith((".cuh", ".h")):
            deps.append(os.path.join(CSRC, name))
    deps.append(os.path.join(ROOT, "include", "tg_gemm.h"))
    return deps


def is_stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(d) > t for d in _deps())


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    if not force and not is_stale():
        return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH, *NVCC_FLAGS, *extra_flags, *SOURCES, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
