"""Builds libattn.so (the C-ABI library in include/attn.h) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libattn.so")
SOURCES = [os.path.join(CSRC, "attn_api.cu"), os.path.join(CSRC, "decode_noalloc.cu"), os.path.join(CSRC, "selftest.cu")]
DEPENDS = SOURCES + [os.path.join(CSRC, f) for f in ("fwd_kernel.cuh", "aux_kernels.cuh", "sm100.cuh")] + [
    os.path.join(ROOT, "include", "attn.h")]

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


# The cycle-trace variant (-DATTN_TRACE): the same kernels with trace records
# at the pipeline hand-offs, plus attn_trace_configure. Used by trace.py only.
TRACE_LIB = os.path.join(HERE, "libattn_trace.so")


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in DEPENDS)


def build(force: bool = False, verbose: bool = False, trace: bool = False) -> str:
    lib = TRACE_LIB if trace else LIB
    if force or stale(lib):
        tmp = lib + ".tmp.%d" % os.getpid()
        cmd = [nvcc()] + NVCC_FLAGS + (["-DATTN_TRACE"] if trace else []) + ["-o", tmp] + SOURCES
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError("nvcc failed building %s" % os.path.basename(lib))
        if verbose:
            sys.stderr.write(res.stderr)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, trace="--trace" in sys.argv))
