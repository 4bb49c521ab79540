"""Builds the in-tree CUDA library ``libpa_b200.so`` for sm_100a with nvcc.

Run ``python -m paged_kv_cache_457_b200.build_lib [--debug]`` (or ``__graft_entry__.build()``, which
builds both).  ``--debug`` builds ``libpa_b200_debug.so`` with PA_DEBUG: the kernels check every index
they derive before using it and report a failed check in the device status word
(PA_DEV_ERR_INTERNAL) instead of touching memory; load it with ``PA_B200_LIBRARY=<path>``.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libpa_b200.so")
# the same sources with PA_DEBUG: every index the kernels derive is checked on the device before use
DEBUG_LIB = os.path.join(PKG, "libpa_b200_debug.so")
SOURCES = [os.path.join(CSRC, "pa_api.cu"), os.path.join(CSRC, "block_manager.cpp"),
           os.path.join(CSRC, "cascade_plan.cpp")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("pa_kernels.cuh", "pa_mma.cuh", "pa_ptx.cuh", "pa_copy.cuh", "pa_prefill.cuh", "pa_tcgen05.cuh", "pa_stream.cuh", "pa_cascade.cuh",
                                                   "pa_plan_layout.h")] + [
    os.path.join(INCLUDE, h) for h in ("pa_b200.h", "pa_block_manager.h")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def command(out: str = LIB, verbose_ptxas: bool = False, debug: bool = False) -> list:
    cmd = [nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-o", out] + SOURCES
    if debug:
        cmd[1:1] = ["-DPA_DEBUG"]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def up_to_date(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False) -> str:
    out = DEBUG_LIB if debug else LIB
    if force or verbose_ptxas or not up_to_date(out):
        subprocess.run(command(out, verbose_ptxas=verbose_ptxas, debug=debug), check=True)
    return out


if __name__ == "__main__":
    debug = "--debug" in sys.argv
    print(build(force=True, verbose_ptxas="-v" in sys.argv, debug=debug))
