"""Compile the CUDA library ``libsla.so`` for sm_100a, in-tree.

    python -m block_sparse_linear_proj_b200.build

One translation unit (``csrc/sla_api.cu`` includes every kernel header), so
the device status word needs no relocatable device code.  The CUDA runtime is
linked statically; the driver is reached at run time.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "sla_api.cu")
LIB = os.path.join(HERE, "libsla.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")


def _sources():
    d = os.path.join(HERE, "csrc")
    out = [os.path.join(d, f) for f in os.listdir(d) if f.endswith((".cu", ".cuh"))]
    out.append(os.path.join(INCLUDE, "sla.h"))
    return out


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(s) <= t for s in _sources()):
            return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE,
           "-diag-suppress", "177", SRC, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas")
        cmd.insert(2, "-v")
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
