"""Compile the C oracle into ``oracle/_build/libbasa_oracle-<host>.so`` with gcc.

Run directly (``python oracle/build.py``) or through ``build_oracle()``.

The oracle is compiled with ``-O3 -march=native`` and OpenMP, so each build is
specific to the CPU it was made on; the file name carries a key of the host's
CPU model and instruction-set flags, and a machine with another CPU builds its
own copy instead of loading one it may not be able to run.  ISO C mode
(``-std=c11``) keeps floating-point contraction off, so ``-march=native``
does not fuse the oracle's multiply-adds.
"""
from __future__ import annotations

import hashlib
import os
import platform
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "basa_oracle.c")
OUT_DIR = os.path.join(HERE, "_build")
FLAGS = ["-O3", "-march=native", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall"]


def host_key() -> str:
    """Short key of this machine's CPU: architecture, model name, ISA flags."""
    parts = [platform.machine()]
    try:
        with open("/proc/cpuinfo") as f:
            seen = set()
            for line in f:
                key = line.split(":", 1)[0].strip()
                if key in ("model name", "flags", "Features") and key not in seen:
                    seen.add(key)
                    parts.append(line.strip())
    except OSError:
        parts.append(platform.processor())
    return hashlib.sha256("\n".join(parts).encode()).hexdigest()[:12]


LIB = os.path.join(OUT_DIR, f"libbasa_oracle-{host_key()}.so")


def build(force: bool = False, verbose: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)
            and os.path.getmtime(LIB) >= os.path.getmtime(__file__)):
        return LIB
    os.makedirs(OUT_DIR, exist_ok=True)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", *FLAGS, "-o", tmp, SRC, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
