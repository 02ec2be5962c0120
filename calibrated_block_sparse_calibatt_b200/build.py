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


def _inputs_digest(trace: bool) -> str:
    """SHA-256 of everything the library is built from: the bytes of every file
    under csrc/ and of the public header, the compiler flags and nvcc's path."""
    import hashlib
    h = hashlib.sha256()
    h.update(repr((ARCH, FLAGS, trace, nvcc())).encode())
    for name in sorted(os.listdir(CSRC)) + [None]:
        path = os.path.join(INCLUDE, "calibatt.h") if name is None else os.path.join(CSRC, name)
        if os.path.isfile(path):
            h.update(os.path.relpath(path, ROOT).encode() + b"\0")
            with open(path, "rb") as f:
                h.update(f.read())
    return h.hexdigest()


def _digest_path(lib: str) -> str:
    return lib + ".inputs-sha256"


def _stale(lib: str = LIB, trace: bool = False) -> bool:
    """True unless the library exists and was built from exactly the current
    sources and flags (content hash recorded beside it at link time).  File
    modification times are not trusted: a copied or unpacked binary can carry
    a newer time than sources it was not built from."""
    if not os.path.exists(lib) or not os.path.exists(_digest_path(lib)):
        return True
    with open(_digest_path(lib)) as f:
        return f.read().strip() != _inputs_digest(trace)


def build(force: bool = False, verbose_ptxas: bool = False, trace: bool = False) -> str:
    """Compiles the library (or, with trace=True, its measurement variant)
    unless it was built from the current sources and flags; returns its path.

    Safe to call from several processes at once (the ranks of a multi-GPU
    run): one builds under an exclusive file lock while the others wait, then
    find the library current; the new file replaces the old one atomically."""
    lib = LIB_TRACE if trace else LIB
    if not force and not verbose_ptxas and not _stale(lib, trace):
        return lib
    os.makedirs(LIBDIR, exist_ok=True)
    with open(os.path.join(LIBDIR, ".build.lock"), "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)
        try:
            if not force and not verbose_ptxas and not _stale(lib, trace):
                return lib                                   # built by another process meanwhile
            digest = _inputs_digest(trace)
            os.makedirs(os.path.join(BUILD, "trace") if trace else BUILD, exist_ok=True)
            with concurrent.futures.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
                objs = list(ex.map(lambda s: _compile(s, verbose_ptxas, trace), SOURCES))
            tmp = f"{lib}.{os.getpid()}.tmp"
            r = subprocess.run([nvcc(), *ARCH, "-shared", "-o", tmp, *objs], capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"link failed:\n{r.stderr}")
            # the digest is written after the library it describes: a crash in
            # between leaves a stale digest, which only forces a rebuild
            if os.path.exists(_digest_path(lib)):
                os.remove(_digest_path(lib))
            os.replace(tmp, lib)
            with open(_digest_path(lib) + ".tmp", "w") as f:
                f.write(digest + "\n")
            os.replace(_digest_path(lib) + ".tmp", _digest_path(lib))
        finally:
            fcntl.flock(lock, fcntl.LOCK_UN)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="-v" in sys.argv))
