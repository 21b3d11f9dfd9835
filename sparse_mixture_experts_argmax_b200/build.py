"""Build libswitchlayer.so (sm_100a) in-tree with nvcc.

Usage: python -m sparse_mixture_experts_argmax_b200.build [--force] [--checked]
Objects go to _build/ at the repository root; the shared library is written
next to this file, where the Python binding loads it.  ``--checked`` builds
libswitchlayer_checked.so with -DSWL_CHECKED: every computed index of the
dispatch and the expert GEMMs is range-checked, a failed check sets the device
status to SWL_ERR_DEVICE and the access is skipped (the binding loads it when
SWL_LIBRARY=checked).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libswitchlayer.so")
LIB_CHECKED = os.path.join(PKG, "libswitchlayer_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "--expt-relaxed-constexpr", "-I" + INCLUDE, "-I" + CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (_sources() + glob.glob(os.path.join(CSRC, "*.h")) +
            glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")) +
            [os.path.abspath(__file__)])


def up_to_date(checked: bool = False) -> bool:
    lib = LIB_CHECKED if checked else LIB
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, extra_flags=(), checked=None) -> str:
    """Compile every CUDA source for sm_100a and link the shared library
    (``checked``: the range-checked variant; None: the one SWL_LIBRARY selects)."""
    if checked is None:
        checked = os.environ.get("SWL_LIBRARY", "") == "checked"
    lib = LIB_CHECKED if checked else LIB
    if not force and up_to_date(checked):
        return lib
    bdir = os.path.join(BUILD, "checked") if checked else BUILD
    os.makedirs(bdir, exist_ok=True)
    nvcc = _nvcc()
    if checked:
        extra_flags = tuple(extra_flags) + ("-DSWL_CHECKED",)

    def compile_one(src):
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [nvcc, *NVCC_FLAGS, *extra_flags, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s%s" % (src, r.stdout, r.stderr))
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, flush=True)
        return obj

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = lib + ".tmp"
    cmd = [nvcc, *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s%s" % (r.stdout, r.stderr))
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    print(build(force="--force" in sys.argv or bool(extra), verbose=True, extra_flags=extra,
                checked="--checked" in sys.argv))
