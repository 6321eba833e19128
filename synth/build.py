"""Build the synthetic-input library ``synth/libsynth.so`` (host twin + device twin).

Run as ``python -m synth.build`` or through ``__graft_entry__.build()``.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libsynth.so")
SRCS = [os.path.join(HERE, "csrc", "synth_host.c"), os.path.join(HERE, "csrc", "synth_dev.cu")]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = SRCS + [os.path.join(HERE, "csrc", "synth.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    cmd = [
        "nvcc", "-O3", "-shared", "-std=c++17",
        "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-fmad=false",
        "-Xcompiler", "-fPIC,-fopenmp,-ffp-contract=off",
        "-I", os.path.join(HERE, "csrc"),
        *SRCS, "-o", LIB, "-lgomp",
    ]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
