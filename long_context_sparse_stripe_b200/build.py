"""Builds libs2o.so in-tree with nvcc for sm_100a (B200).

Index kernels compile with ``--fmad=false`` (every rounding there is explicit anyway) and
without fast-math, so the index arrays match the definition bit for bit; the attention kernel
compiles with ``-O3``. Used by ``__graft_entry__.build()`` and on first import of the package.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libs2o.so")
BUILD = os.path.join(ROOT, "_build")

SOURCES = {
    "s2o_api.cu": ["-O3"],
    "s2o_index.cu": ["-O3", "--fmad=false", "-ftz=false", "-prec-div=true", "-prec-sqrt=true"],
    "s2o_attn.cu": ["-O3"],
    "s2o_static_ws.cu": ["-O3"],
    "s2o_layer.cu": ["-O3"],
    "s2o_gemm.cu": ["-O3"],
}
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(ROOT, "include", "s2o.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    objs = []
    common = [nvcc(), *ARCH, "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC",
              "-I", os.path.join(ROOT, "include"), "-I", CSRC]
    if verbose:
        common += ["-Xptxas", "-v"]
    for src, flags in SOURCES.items():
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        cmd = [*common, *flags, "-c", os.path.join(CSRC, src), "-o", obj]
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static",
                    "-ldl", "-lrt", "-lpthread"], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
