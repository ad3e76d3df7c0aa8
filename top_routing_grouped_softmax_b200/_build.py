"""Build libmoe.so (the C-ABI library) from csrc/ with nvcc for sm_100a.

The library is rebuilt when the sources, the public header or the flags
change (a content hash is stored next to it), so a stale binary is never
loaded.  nvcc cross-compiles without a GPU.
"""
from __future__ import annotations

import glob
import hashlib
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmoe.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
    "--expt-relaxed-constexpr",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  [os.path.join(INCLUDE, "moe.h")])


def _hash(flags) -> str:
    h = hashlib.sha256()
    for p in _sources():
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as fh:
            h.update(fh.read())
    h.update(" ".join(flags).encode())
    return h.hexdigest()


def kernel_hash(files=("grouped_gemm.cuh", "grouped_gemm_pair.cuh", "ptx.cuh", "status.cuh")) -> str:
    """Hash of the grouped-GEMM kernel sources and the build flags: ties a
    profiler measurement to the kernel version it was taken on."""
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(CSRC, name), "rb") as fh:
            h.update(fh.read())
    h.update(" ".join(NVCC_FLAGS).encode())
    return h.hexdigest()[:16]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build_library(force: bool = False, verbose: bool = False, out: str = LIB, extra_flags=()) -> str:
    flags = NVCC_FLAGS + list(extra_flags)
    stamp = out + ".srchash"
    digest = _hash(flags)
    if not force and os.path.exists(out) and os.path.exists(stamp):
        with open(stamp) as fh:
            if fh.read().strip() == digest:
                return out
    cmd = [nvcc(), *flags, "-I", INCLUDE, "-I", CSRC, "-o", out, os.path.join(CSRC, "moe.cu")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        print(res.stdout + res.stderr)
    with open(os.path.join(PKG, "ptxas_info.txt"), "w") as fh:
        fh.write(res.stderr)
    with open(stamp, "w") as fh:
        fh.write(digest)
    return out


if __name__ == "__main__":
    build_library(force=True, verbose=True)
