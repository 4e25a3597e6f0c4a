"""Build ``libdeltakv.so`` in-tree for B200 (sm_100a) with nvcc.

The library is the CUDA translation unit ``csrc/deltakv.cu`` plus the host-only ``csrc/pool.cpp`` (block pool
and batching planner), with the CUDA runtime linked statically and
the driver's tensor-map encoder resolved at run time, so the shared object loads on a host without a
GPU driver (the symbol-export tests need that).  Usage: ``python -m residual_kv_cache_delta_b200.build``.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
# the CUDA translation unit (kernels + C ABI) and the host-only block pool / batching planner
SRCS = [os.path.join(HERE, "csrc", "deltakv.cu"), os.path.join(HERE, "csrc", "pool.cpp")]
OUT = os.path.join(HERE, "libdeltakv.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
         "-shared", "-cudart", "static"]


def sources() -> list[str]:
    d = os.path.join(HERE, "csrc")
    inc = os.path.join(HERE, "..", "include")
    return [os.path.join(d, f) for f in sorted(os.listdir(d))] + [os.path.join(inc, f) for f in sorted(os.listdir(inc))]


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    if not force and not extra and up_to_date():
        return OUT
    cmd = [NVCC, *FLAGS, *(extra or []), "-o", OUT, *SRCS]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return OUT


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
