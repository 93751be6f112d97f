"""Builds libsdpa.so in-tree: every .cu under csrc/ compiled by nvcc for sm_100a only.

    python head_scaled_dot_sdpa_b200/build.py [--force] [--debug-checks]

With --debug-checks (or build(debug_checks=True)) the same sources are compiled with
-DSDPA_DEBUG_CHECKS into libsdpa_debug.so: every device-side index the kernels take from data
(block lists and counts, partial-bit addresses, TMA tile coordinates, cache and split indices,
output rows) is range-checked in the kernel; a violation records SDPA_ERR_DEVICE_CHECK in the
status word and the access is skipped or clamped, never trapped. The package loads that
library instead of libsdpa.so when the environment has SDPA_DEBUG_CHECKS=1.

(run as a file, so that the package, which loads the library, is not imported first)

The CUDA runtime is linked statically and the driver API (used for TMA descriptors) is
looked up at run time, so the library loads on a machine without a GPU driver.
"""
from __future__ import annotations

import concurrent.futures
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build", "sdpa")
LIB = os.path.join(PKG, "libsdpa.so")
BUILD_DEBUG = os.path.join(ROOT, "_build", "sdpa_debug")
LIB_DEBUG = os.path.join(PKG, "libsdpa_debug.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps():
    return [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "sdpa.h")]


def _compile(src: str, verbose: bool, debug_checks: bool = False) -> str:
    obj = os.path.join(BUILD_DEBUG if debug_checks else BUILD, os.path.basename(src) + ".o")
    newest = max(os.path.getmtime(d) for d in _deps())
    if os.path.exists(obj) and os.path.getmtime(obj) >= newest:
        return obj
    cmd = [NVCC, *ARCH, *FLAGS, *(["-DSDPA_DEBUG_CHECKS"] if debug_checks else []), "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{res.stderr}")
    if verbose and res.stderr:
        sys.stderr.write(res.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, debug_checks: bool = False) -> str:
    bdir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug_checks else (BUILD, LIB)
    os.makedirs(bdir, exist_ok=True)
    if force:
        for f in os.listdir(bdir):
            os.remove(os.path.join(bdir, f))
    srcs = _sources()
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, debug_checks), srcs))
    newest = max(os.path.getmtime(o) for o in objs)
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < newest:
        tmp = lib + ".tmp"
        cmd = [NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-cudart", "static", "-o", tmp, *objs]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"link failed:\n{res.stderr}")
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug_checks="--debug-checks" in sys.argv))
