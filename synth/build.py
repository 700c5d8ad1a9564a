"""Builds the seeded input generator: a host library (gcc, OpenMP) and a device
library (nvcc, sm_100a).  Both compile the one header ``philox.h``."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(HERE, "libsynth_host.so")
DEV_SO = os.path.join(HERE, "libsynth_dev.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _run(cmd):
    print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build(force: bool = False) -> None:
    hdr = os.path.join(HERE, "philox.h")
    src_h = os.path.join(HERE, "synth_host.c")
    src_d = os.path.join(HERE, "synth_dev.cu")
    if force or _stale(HOST_SO, [hdr, src_h]):
        _run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
              "-fno-fast-math", "-o", HOST_SO, src_h, "-lm"])
    if force or _stale(DEV_SO, [hdr, src_d]):
        _run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
              "--fmad=false", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
              "-Xcompiler", "-fPIC", "-shared", "-o", DEV_SO, src_d])


if __name__ == "__main__":
    build(force="--force" in sys.argv)
