"""Build libzb.so (the sm_100a device library) in-tree with nvcc.

    python -m token_dispatch_top_b200.build [--force] [--debug]

Compiles every ``csrc/*.cu`` for sm_100a only, without fast-math (the combine
relies on IEEE fused multiply-add and round-to-nearest-even conversions), and
links the CUDA runtime statically so the library needs only the driver.
``--debug`` builds libzb_debug.so instead: the same kernels with -DZB_DEBUG,
whose data-indexed accesses are bounds-checked and whose failed checks are
recorded for zb_debug_read.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libzb.so")
LIB_DEBUG = os.path.join(HERE, "libzb_debug.so")
INCLUDE = os.path.join(ROOT, "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=true",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-cudart", "static",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def _deps() -> list[str]:
    return sources() + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + \
        [os.path.join(INCLUDE, "zb.h"), __file__]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    flags = NVCC_FLAGS + (["-DZB_DEBUG"] if debug else [])
    cmd = [nvcc, *flags, "-I", INCLUDE, "-shared", "-o", tmp, *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                debug="--debug" in sys.argv))
