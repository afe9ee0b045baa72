"""Builds the CUDA library ``libjetfire.so`` in-tree with nvcc for sm_100a.

Run as ``python -m int8_fully_quantized_b200.build_lib`` (or through ``__graft_entry__.build()``).
The build needs only nvcc (it cross-compiles without a GPU). No fast-math flags are used: the
quantizer relies on IEEE division, reciprocal and denormal handling.
"""
from __future__ import annotations

import glob
import hashlib
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG_DIR, "libjetfire.so")
HASH_PATH = LIB_PATH + ".srchash"
# The same sources with NVTX ranges around every compute entry point (-DJF_NVTX), for profiling with
# a tool that records NVTX; load it with JETFIRE_LIB=<this path>. The product library has no ranges.
NVTX_LIB_PATH = os.path.join(PKG_DIR, "libjetfire_nvtx.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "-shared", "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libjetfire.so")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]


def source_hash() -> str:
    """Content hash of every file the library is built from (sources, headers, this script)."""
    h = hashlib.sha256()
    for p in sorted(_inputs()):
        h.update(os.path.relpath(p, ROOT).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


# Files that define the block-scaled GEMM kernel's device code (its host launcher lives in gemm.cu too).
GEMM_KERNEL_FILES = ("gemm.cu", "ptx.cuh", "quant.cuh", "act.cuh")


def kernel_source_hash(names=GEMM_KERNEL_FILES) -> str:
    """Content hash of the given csrc files only: a record taken of one kernel (e.g. its ncu DRAM
    traffic) stays valid while these files are unchanged, whatever else in the library changes."""
    h = hashlib.sha256()
    for n in sorted(names):
        h.update(n.encode())
        with open(os.path.join(CSRC, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def built_hash() -> str | None:
    try:
        with open(HASH_PATH) as f:
            return f.read().strip()
    except OSError:
        return None


def up_to_date() -> bool:
    return os.path.exists(LIB_PATH) and built_hash() == source_hash()


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None) -> str:
    """Compile every ``csrc/*.cu`` into ``libjetfire.so`` (skipped when up to date)."""
    if not force and up_to_date():
        return LIB_PATH
    tmp = LIB_PATH + ".tmp"
    cmd = [_nvcc(), *ARCH_FLAGS, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, *(extra_flags or []),
           *sources(), "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr, file=sys.stderr)
    os.replace(tmp, LIB_PATH)
    with open(HASH_PATH, "w") as f:
        f.write(source_hash())
    return LIB_PATH


def build_nvtx(verbose: bool = False) -> str:
    """Compile the instrumented variant (NVTX ranges, -DJF_NVTX) into ``libjetfire_nvtx.so``."""
    tmp = NVTX_LIB_PATH + ".tmp"
    cmd = [_nvcc(), *ARCH_FLAGS, *NVCC_FLAGS, "-DJF_NVTX", "-I", INCLUDE, "-I", CSRC, *sources(), "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, NVTX_LIB_PATH)
    return NVTX_LIB_PATH


if __name__ == "__main__":
    if "--nvtx" in sys.argv:
        print(build_nvtx(verbose=True))
    else:
        print(build(force="--force" in sys.argv, verbose=True,
                    extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None))
