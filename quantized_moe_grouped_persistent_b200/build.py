"""Compile the sm_100a CUDA libraries in-tree: quantized_moe_grouped_persistent_b200/libqgmm.so
(the op, with the expert-parallel dispatch plan) and libqgmm_probe.so (the int8 tensor-rate probe the benchmark reads its roofline against)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libqgmm.so")
MAIN = [os.path.join(HERE, "csrc", "qgmm.cu"), os.path.join(HERE, "csrc", "ep_plan.cu"),
        os.path.join(HERE, "csrc", "ep_permute.cu")]
PROBE_LIB = os.path.join(HERE, "libqgmm_probe.so")
PROBE = [os.path.join(HERE, "csrc", "probe_mma.cu")]
NVCC_FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared",
]


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*"))) + sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


def _compile(srcs: list, lib: str, force: bool, verbose: bool) -> str:
    if not force and os.path.exists(lib):
        newest = max(os.path.getmtime(s) for s in sources())
        if os.path.getmtime(lib) >= newest:
            return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *(["-Xptxas", "-v"] if verbose else []), *srcs, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    _compile(PROBE, PROBE_LIB, force, verbose)
    return _compile(MAIN, LIB, force, verbose)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
