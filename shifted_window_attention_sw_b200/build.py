"""Build ``libvswin.so`` (the CUDA library behind ``include/vswin.h``) in-tree.

nvcc compiles every ``csrc/*.cu`` for sm_100a only and links the CUDA runtime
statically, so the library loads on any machine with the same driver stack
(and also loads, without running kernels, on a machine with no GPU).

    python -m shifted_window_attention_sw_b200.build [--force] [--verbose]
"""

from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libvswin.so")
# the same library with VSWIN_DEBUG_BOUNDS: every gather / scatter index of the
# row tables checked against its extent (a violation sets the error word and
# skips the access)
LIB_DEBUG = os.path.join(PKG, "libvswin_debug.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
              "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libvswin.so")
    return exe


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + [
        os.path.join(ROOT, "include", "vswin.h")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug_bounds: bool = False) -> str:
    lib = LIB_DEBUG if debug_bounds else LIB
    if not force and up_to_date(lib):
        return lib
    bdir = os.path.join(BUILD_DIR, "debug_bounds") if debug_bounds else BUILD_DIR
    os.makedirs(bdir, exist_ok=True)
    exe = nvcc()
    flags = [*NVCC_FLAGS, *(["-DVSWIN_DEBUG_BOUNDS"] if debug_bounds else []), *extra_flags]

    def compile_one(src):
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [exe, *ARCH, *flags, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, file=sys.stderr)
        return obj

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [exe, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas resource usage")
    ap.add_argument("--debug-bounds", action="store_true", help="build libvswin_debug.so (VSWIN_DEBUG_BOUNDS)")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, debug_bounds=args.debug_bounds))
