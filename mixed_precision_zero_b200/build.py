"""Build the CUDA library in-tree with nvcc for sm_100a (B200).

    python -m mixed_precision_zero_b200.build

writes ``mixed_precision_zero_b200/libneoxshard.so``.  No fast-math: IEEE
division and square root, and explicit round-to-nearest intrinsics in the
kernels where the order of FP32 operations is part of the result.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
INCLUDE = os.path.join(ROOT, "include")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared",
                     "-Xptxas", "-v", "-I", INCLUDE]

SOURCES = [os.path.join(PKG, "csrc", f) for f in ("neox_shard.cu", "neox_multi.cu", "neox_peer.cu")]
LIB = os.path.join(PKG, "libneoxshard.so")


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    deps = SOURCES + [os.path.join(INCLUDE, "neox_shard.h"), os.path.join(PKG, "csrc", "neox_common.cuh")]
    if force or _stale(LIB, deps):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [NVCC, *NVCC_FLAGS, "-o", tmp, *SOURCES]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError(f"nvcc failed ({res.returncode}) building {LIB}")
        if verbose:
            sys.stderr.write(res.stderr)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
