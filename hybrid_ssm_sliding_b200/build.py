"""Builds libsamba.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m hybrid_ssm_sliding_b200.build [--force] [--verbose] [--debug]

Each csrc/*.cu file is compiled on its own (in parallel) and the objects are
linked into hybrid_ssm_sliding_b200/libsamba.so with the static CUDA runtime,
so the library needs nothing at run time beyond the driver.  ``--debug``
builds libsamba_debug.so instead: the same sources with SAMBA_DEBUG, whose
kernels check every global output store's index and report a failed check
in the status word (SAMBA_ERR_CHECK) instead of storing.
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libsamba.so")
OBJ_DEBUG = os.path.join(PKG, "_build_debug")
LIB_DEBUG = os.path.join(PKG, "libsamba_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA library cannot be built")
    return path


def _deps() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*"))) + [os.path.join(ROOT, "include", "samba.h")]


def source_hash() -> str:
    """Short hash of the CUDA sources and the header (ties profiles to code)."""
    import hashlib

    h = hashlib.sha256()
    for d in _deps():
        if os.path.isfile(d):
            h.update(os.path.basename(d).encode())
            with open(d, "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:12]


def kernel_hash(name: str) -> str:
    """Short hash of one kernel file (``csrc/<name>.cu``) and the shared device
    header it includes: the sources that fix that kernel's device code, so a
    recorded profile of it stays valid while other files change."""
    import hashlib

    h = hashlib.sha256()
    for d in (os.path.join(CSRC, name + ".cu"), os.path.join(CSRC, "common.cuh")):
        h.update(os.path.basename(d).encode())
        with open(d, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = False) -> str:
    """Builds libsamba.so (or, with ``debug``, libsamba_debug.so) unless it
    is newer than every source; returns its path."""
    lib, obj_dir = (LIB_DEBUG, OBJ_DEBUG) if debug else (LIB, OBJ)
    if debug:
        extra = (*extra, "-DSAMBA_DEBUG")
    if not force and up_to_date(lib):
        return lib
    os.makedirs(obj_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    cc = nvcc()

    def compile_one(src: str) -> str:
        obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
        cmd = [cc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stderr[-6000:]}")
        if verbose and r.stderr:
            sys.stderr.write(r.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, len(sources))) as ex:
        objs = list(ex.map(compile_one, sources))
    tmp = lib + ".tmp"
    cmd = [cc, *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr[-4000:]}")
    os.replace(tmp, lib)
    return lib


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/spill reports")
    ap.add_argument("--debug", action="store_true", help="build libsamba_debug.so (device-side index checks)")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, debug=a.debug))


if __name__ == "__main__":
    main()
