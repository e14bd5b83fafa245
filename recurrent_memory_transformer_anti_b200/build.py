"""Build librmt.so (sm_100a) in place with nvcc: one object per source, linked shared.

Also builds librmt_debug.so, the same sources compiled with -DRMT_DEBUG: every kernel checks
the indices it takes from its cell table against the buffers they address and reports a
violation through the error word (rmt_sync: RMT_EDEBUG) instead of making the access.

Run as `python -m recurrent_memory_transformer_anti_b200.build [--force] [--debug]`.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJDIR = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "librmt.so")
OBJDIR_DEBUG = os.path.join(PKG, "_build_debug")
LIB_DEBUG = os.path.join(PKG, "librmt_debug.so")
SOURCES = ["api.cu", "tc_gemm.cu", "tc_gemm_pair.cu", "simt_gemm.cu", "attention.cu", "attention_tc.cu", "memory.cu", "memory_tc.cu", "rowops.cu", "noalloc.cu",
           "selftest.cu"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]


def _deps_mtime() -> float:
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "rmt.h")]
    return max(os.path.getmtime(f) for f in files)


def _compile(src: str, extra: list, objdir: str) -> str:
    obj = os.path.join(objdir, src.replace(".cu", ".o"))
    cmd = [NVCC, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
    if r.stderr.strip():
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, extra_flags: list | None = None, debug: bool = False) -> str:
    """Compile every CUDA source for sm_100a and link librmt.so (librmt_debug.so with debug);
    skip if up to date."""
    objdir, lib = (OBJDIR_DEBUG, LIB_DEBUG) if debug else (OBJDIR, LIB)
    os.makedirs(objdir, exist_ok=True)
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= _deps_mtime():
        return lib
    extra = list(extra_flags or []) + (["-DRMT_DEBUG"] if debug else [])
    with cf.ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 4)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, objdir), SOURCES))
    tmp = lib + ".tmp"
    r = subprocess.run([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", tmp],
                       capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None,
                debug="--debug" in sys.argv))
