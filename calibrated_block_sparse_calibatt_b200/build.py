"""Builds libcalibatt.so in-tree with nvcc for sm_100a (B200).

Each CUDA source compiles to an object under <repo>/_build, then everything
links into calibrated_block_sparse_calibatt_b200/lib/libcalibatt.so with the
CUDA runtime linked statically (the driver is loaded when first used, so the
library also loads on a machine without a GPU).
"""

from __future__ import annotations

import concurrent.futures
import fcntl
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libcalibatt.so")
BUILD = os.path.join(ROOT, "_build")
# Measurement variant: the same sources with -DCALIBATT_TRACE (pipeline and
# epilogue timers compiled in); never loaded by the product path.
LIB_TRACE = os.path.join(LIBDIR, "libcalibatt_trace.so")

SOURCES = ["api.cu", "attn_tc.cu", "attn_simt.cu", "energy.cu", "energy_noalloc.cu", "repetition.cu",
           "diagnostics.cu", "csr_check.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _compile(src: str, verbose_ptxas: bool, trace: bool = False) -> str:
    obj = os.path.join(BUILD, "trace" if trace else "", src.replace(".cu", ".o"))
    cmd = [nvcc(), *ARCH, *FLAGS, *(["-DCALIBATT_TRACE"] if trace else []), "-c", os.path.join(CSRC, src),
           "-o", obj]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    return obj


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "calibatt.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False, trace: bool = False) -> str:
    """Compiles the library (or, with trace=True, its measurement variant) if
    any source is newer than it; returns its path.

    Safe to call from several processes at once (the ranks of a multi-GPU
    run): one builds under an exclusive file lock while the others wait, then
    find the library current; the new file replaces the old one atomically."""
    lib = LIB_TRACE if trace else LIB
    if not force and not verbose_ptxas and not _stale(lib):
        return lib
    os.makedirs(LIBDIR, exist_ok=True)
    with open(os.path.join(LIBDIR, ".build.lock"), "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)
        try:
            if not force and not verbose_ptxas and not _stale(lib):
                return lib                                   # built by another process meanwhile
            os.makedirs(os.path.join(BUILD, "trace") if trace else BUILD, exist_ok=True)
            with concurrent.futures.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
                objs = list(ex.map(lambda s: _compile(s, verbose_ptxas, trace), SOURCES))
            tmp = f"{lib}.{os.getpid()}.tmp"
            r = subprocess.run([nvcc(), *ARCH, "-shared", "-o", tmp, *objs], capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"link failed:\n{r.stderr}")
            os.replace(tmp, lib)
        finally:
            fcntl.flock(lock, fcntl.LOCK_UN)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="-v" in sys.argv))
