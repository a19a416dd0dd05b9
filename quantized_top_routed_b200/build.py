"""Build libqmoe.so in-tree with nvcc for sm_100a (B200).

``python -m quantized_top_routed_b200.build [--force] [--verbose]``

Objects go to ``_build/`` at the repository root; the shared libraries are
written next to this file.  The CUDA runtime is linked statically, so the
library only needs the NVIDIA driver at run time.

Two libraries are built from the same sources: ``libqmoe.so`` and
``libqmoe_debug.so`` (``-DQMOE_DEBUG``: device-side bounds checks that raise
QMOE_ERR_BOUNDS instead of faulting).  The binding loads the second only
when the environment sets ``QMOE_DEBUG=1``.
"""
from __future__ import annotations

import argparse
import concurrent.futures
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libqmoe.so")
LIB_DEBUG = os.path.join(PKG, "libqmoe_debug.so")
SOURCES = ["api.cu", "router.cu", "schedule.cu", "gemm.cu", "combine.cu", "repack.cu"]
HEADERS = ["qmoe_internal.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA toolkit is needed to build libqmoe.so")


def _inputs():
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "qmoe.h"))
    deps.append(os.path.abspath(__file__))
    return deps


HASH = LIB + ".srchash"


def _flags(debug: bool):
    return FLAGS + (["-DQMOE_DEBUG"] if debug else [])


def source_hash(debug: bool = False) -> str:
    h = hashlib.sha256()
    for p in _inputs():
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(f.read())
    h.update(" ".join(ARCH + _flags(debug)).encode())
    return h.hexdigest()


def up_to_date(debug: bool = False) -> bool:
    """The library exists and was built from exactly the current sources
    (content hash, so copies of the tree with fresh timestamps still match)."""
    lib = LIB_DEBUG if debug else LIB
    if not (os.path.exists(lib) and os.path.exists(lib + ".srchash")):
        return False
    with open(lib + ".srchash") as f:
        return f.read().strip() == source_hash(debug)


def _compile(src: str, verbose: bool, debug: bool = False) -> str:
    obj = os.path.join(BUILD, "debug" if debug else "", os.path.splitext(src)[0] + ".o")
    cmd = [nvcc(), *ARCH, *_flags(debug), "-c", os.path.join(CSRC, src), "-o", obj]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(debug):
        return lib
    os.makedirs(os.path.join(BUILD, "debug" if debug else ""), exist_ok=True)
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, debug), SOURCES))
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    with open(lib + ".srchash", "w") as f:
        f.write(source_hash(debug))
    return lib


def build_all(force: bool = False, verbose: bool = False) -> list:
    """Both libraries: the product one and the QMOE_DEBUG one."""
    return [build(force, verbose, debug=False), build(force, verbose, debug=True)]


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/smem usage")
    ap.add_argument("--debug-only", action="store_true", help="build only libqmoe_debug.so")
    ap.add_argument("--product-only", action="store_true", help="build only libqmoe.so")
    args = ap.parse_args()
    if not args.product_only:
        print(build(force=args.force, verbose=args.verbose, debug=True))
    if not args.debug_only:
        print(build(force=args.force, verbose=args.verbose))
