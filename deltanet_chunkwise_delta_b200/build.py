"""Builds the sm_100a shared library behind the C ABI (include/deltanet.h).

``python -m deltanet_chunkwise_delta_b200.build`` compiles ``csrc/deltanet.cu``
and ``csrc/deltanet_noalloc.cu`` with nvcc into ``_build/libdeltanet_b200.so``
inside the package directory, so the library travels with the source tree.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRCS = [os.path.join(PKG, "csrc", "deltanet.cu"), os.path.join(PKG, "csrc", "deltanet_noalloc.cu")]
LIB = os.path.join(PKG, "_build", "libdeltanet_b200.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC",
    "-Xptxas", "-v",
]


def _sources():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*"))) + \
        [os.path.join(ROOT, "include", "deltanet.h")]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, "-o", tmp, *SRCS]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    log = os.path.join(os.path.dirname(LIB), "ptxas.log")
    with open(log, "w") as f:
        f.write(res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
