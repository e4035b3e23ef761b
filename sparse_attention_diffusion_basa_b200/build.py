"""Build the C-ABI shared library ``_lib/libbasa.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m sparse_attention_diffusion_basa_b200.build [--force] [--verbose]
[--checked]``.  The library links the CUDA runtime statically and resolves the
TMA map encoder through the driver entry point, so it loads on machines without
a GPU.  ``--checked`` builds ``_lib/libbasa_checked.so`` instead: the same
library compiled with BASA_CHECKED, whose kernels check every TMA box and every
output index against their tensors, skip an access that is out of range and
report it through the device status word (BASA_ERR_CHECK); the binding loads it
when the environment variable BASA_LIBRARY is ``checked``.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OUT_DIR = os.path.join(HERE, "_lib")
LIB = os.path.join(OUT_DIR, "libbasa.so")
LIB_CHECKED = os.path.join(OUT_DIR, "libbasa_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = (sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))
    return any(os.path.getmtime(f) > t for f in deps)


def build(force: bool = False, verbose: bool = False, extra=(), checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    if not force and not _stale(lib):
        return lib
    os.makedirs(OUT_DIR, exist_ok=True)
    tmp = lib + f".tmp{os.getpid()}"
    flags = [*NVCC_FLAGS, *extra] + (["-DBASA_CHECKED"] if checked else [])
    cmd = [_nvcc(), *flags, "-I", INCLUDE, "-I", CSRC, "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    extra = ["-Xptxas", "-v"] if "--ptxas" in sys.argv else []
    print(build(force="--force" in sys.argv or bool(extra), verbose="--verbose" in sys.argv,
                extra=extra, checked="--checked" in sys.argv))
