"""Build the CUDA library ``libeqlin.so`` in-tree for sm_100a with nvcc.

Usage: ``python -m group_circulant_linear_b200.build [--force]``.  The
library links only the CUDA runtime (static) so that it loads on machines
without a GPU driver; the driver entry points it needs (tensor-map encoding)
are looked up at run time.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libeqlin.so")
SOURCES = ["eqlin_api.cu", "eqlin_simt.cu", "eqlin_tc.cu", "eqlin_tc32.cu", "eqlin_tc32_dw.cu", "eqlin_tc_dw.cu", "eqlin_tc_dws.cu",
           "eqlin_dihedral.cu", "eqlin_noalloc.cu"]
HEADERS = ["eqlin_internal.cuh", "eqlin_ptx.cuh", "eqlin_packed.cuh", "eqlin_wait.cuh"]
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-cudart", "static",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.join(INCLUDE, "eqlin.h")]
    return any(os.path.exists(d) and os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        cmd = [_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([_nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-cudart", "static", *objs, "-o", tmp, "-ldl", "-lrt", "-lpthread"], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
