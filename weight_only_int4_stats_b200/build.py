"""Builds libawq_b200.so in place (sm_100a only), and its bounds-checking debug twin.

    python -m weight_only_int4_stats_b200.build [--verbose-ptxas] [--debug | --trace]

nvcc cross-compiles without a GPU. The CUDA runtime is linked statically and the driver's
tensor-map encoder is looked up at run time, so the library loads on a machine without a
GPU (every call then returns AWQ_ERR_CUDA).

The debug build (libawq_b200_debug.so, -DAWQ_DEBUG_BOUNDS) compiles index checks into the
kernels: an access whose index falls outside the extent the shapes give is skipped and
recorded in the device status word, which awq_check_error reports as AWQ_ERR_BOUNDS. It is a
stand-in for a memory checker, used by the tests; the release build has no such checks.

The trace build (libawq_b200_trace.so, -DAWQ_TRACE) records a %globaltimer timeline of the
streaming decode kernel's CTAs (awq_trace_read); `bench.py --only trace` prints its summary.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libawq_b200.so")
LIB_DEBUG = os.path.join(PKG, "libawq_b200_debug.so")
LIB_TRACE = os.path.join(PKG, "libawq_b200_trace.so")
SOURCES = [os.path.join(PKG, "csrc", "awq_api.cu")]
DEPS = [os.path.join(PKG, "csrc", f) for f in os.listdir(os.path.join(PKG, "csrc"))] + [
    os.path.join(ROOT, "include", "awq.h")]


def nvcc_path() -> str:
    p = shutil.which("nvcc")
    if p:
        return p
    p = "/usr/local/cuda/bin/nvcc"
    if os.path.exists(p):
        return p
    raise RuntimeError("nvcc not found")


def _path(debug: bool, trace: bool) -> str:
    return LIB_TRACE if trace else LIB_DEBUG if debug else LIB


def command(verbose_ptxas: bool = False, debug: bool = False, trace: bool = False) -> list[str]:
    cmd = [
        nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
        "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
        "-I", os.path.join(ROOT, "include"), "-I", os.path.join(PKG, "csrc"),
        "-o", _path(debug, trace),
    ] + SOURCES
    if debug:
        cmd[1:1] = ["-DAWQ_DEBUG_BOUNDS=1"]
    if trace:
        cmd[1:1] = ["-DAWQ_TRACE=1"]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def up_to_date(path: str = LIB) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(d) <= t for d in DEPS if os.path.exists(d))


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False,
          trace: bool = False) -> str:
    path = _path(debug, trace)
    if force or verbose_ptxas or not up_to_date(path):
        subprocess.run(command(verbose_ptxas, debug, trace), check=True)
    return path


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv,
                debug="--debug" in sys.argv, trace="--trace" in sys.argv))
