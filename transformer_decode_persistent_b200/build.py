"""Build the decode library in-tree with nvcc for sm_100a (B200).

Two libraries from the same sources: libkie.so (the product) and
libkie_trace.so (compiled with KIE_TRACE: the kernel also stamps the start,
input-ready, tiles-done and epilogue-done times of every phase into the
caller's trace buffer; used for measurement only).

Usage: python -m transformer_decode_persistent_b200.build [--verbose]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libkie.so")
LIB_TRACE = os.path.join(HERE, "libkie_trace.so")
SOURCES = ["monokernel.cu", "kie_host.cu", "prefill.cu"]
HEADERS = ["kie_internal.h", "prefill.h", os.path.join("..", "..", "include", "kie.h")]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.abspath(__file__)]
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def _build_one(lib: str, defines, verbose: bool, force: bool, ptxas_info: bool) -> str:
    if not force and not _stale(lib):
        return lib
    tmp = lib + f".{os.getpid()}.tmp"
    cmd = [nvcc(), *ARCH, *FLAGS, *defines, "-shared", "-o", tmp,
           *[os.path.join(CSRC, s) for s in SOURCES]]
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose or ptxas_info:
        sys.stdout.write(r.stdout + r.stderr)
    os.replace(tmp, lib)
    return lib


def build(verbose: bool = False, force: bool = False, ptxas_info: bool = False) -> str:
    """Compile the CUDA sources into libkie.so and libkie_trace.so next to this
    file; returns the product library's path."""
    _build_one(LIB, [], verbose, force, ptxas_info)
    _build_one(LIB_TRACE, ["-DKIE_TRACE"], verbose, force, False)
    return LIB


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force="--force" in sys.argv,
          ptxas_info="--ptxas-info" in sys.argv)
    print(LIB)
