"""Build the decode library in-tree with nvcc for sm_100a (B200).

Two libraries from the same sources: libkie.so (the product) and
libkie_trace.so (compiled with KIE_TRACE: the kernel also stamps the start,
input-ready, tiles-done and epilogue-done times of every phase into the
caller's trace buffer; used for measurement only).

The decode kernel is compiled once per head_dim (128, 64) and FFN kind (dense,
MoE) from decode_inst.cu; the translation units are compiled in parallel and
linked into one shared library.

Usage: python -m transformer_decode_persistent_b200.build [--verbose]
"""
from __future__ import annotations

import concurrent.futures
import os
import shutil
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libkie.so")
LIB_TRACE = os.path.join(HERE, "libkie_trace.so")
SOURCES = ["decode_inst.cu", "kie_host.cu", "prefill.cu"]
HEADERS = ["monokernel.cuh", "kie_internal.h", "prefill.h", os.path.join("..", "..", "include", "kie.h")]
# (source, defines): one decode-kernel unit per (head_dim, MoE), then the host side
UNITS = [("decode_inst.cu", ["-DKIE_DH=128", "-DKIE_MOE=0"]), ("decode_inst.cu", ["-DKIE_DH=128", "-DKIE_MOE=1"]),
         ("decode_inst.cu", ["-DKIE_DH=64", "-DKIE_MOE=0"]), ("decode_inst.cu", ["-DKIE_DH=64", "-DKIE_MOE=1"]),
         ("kie_host.cu", []), ("prefill.cu", [])]

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


def _run(cmd, verbose: bool):
    if verbose:
        print(" ".join(cmd), flush=True)
    return subprocess.run(cmd, capture_output=True, text=True)


def _build_one(lib: str, defines, verbose: bool, force: bool, ptxas_info: bool) -> str:
    if not force and not _stale(lib):
        return lib
    tmp = lib + f".{os.getpid()}.tmp"
    with tempfile.TemporaryDirectory(prefix="kie_build_") as objdir:
        cmds = []
        for n, (src, unit_defs) in enumerate(UNITS):
            obj = os.path.join(objdir, f"{n}_{os.path.splitext(src)[0]}.o")
            cmd = [nvcc(), *ARCH, *FLAGS, *defines, *unit_defs, "-c", "-o", obj, os.path.join(CSRC, src)]
            if ptxas_info:
                cmd.insert(1, "-Xptxas=-v")
            cmds.append((cmd, obj))
        with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, min(len(cmds), os.cpu_count() or 1))) as ex:
            results = list(ex.map(lambda c: _run(c[0], verbose), cmds))
        for (cmd, _), r in zip(cmds, results):
            if r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
                raise RuntimeError(f"nvcc failed building {os.path.basename(lib)} ({cmd[-1]})")
            if verbose or ptxas_info:
                sys.stdout.write(r.stdout + r.stderr)
        r = _run([nvcc(), *ARCH, "-shared", "-o", tmp, *[o for _, o in cmds]], verbose)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"nvcc failed linking {os.path.basename(lib)}")
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
