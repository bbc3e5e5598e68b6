"""Build libmoefp8.so in-tree with nvcc for sm_100a (B200).

    python -m mixture_experts_fp8_b200.build [--force] [--verbose]

Each .cu under csrc/ is compiled to an object under _build/ (in parallel, skipped when up to
date) and linked with the static CUDA runtime into mixture_experts_fp8_b200/libmoefp8.so.
`--debug` (or build_all()) also builds libmoefp8_debug.so from the same sources with
MOE_FAULT_INJECTION, the library the failure-detection tests inject faults through.  The
driver API entry point used for TMA descriptors is fetched at run time, so the library does not
link libcuda.
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
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libmoefp8.so")
# The debug library: the same sources with MOE_FAULT_INJECTION, for failure-detection tests.
BUILD_DEBUG = os.path.join(PKG, "_build_debug")
LIB_DEBUG = os.path.join(PKG, "libmoefp8_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
              "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmoefp8.so")
    return exe


def _deps_mtime() -> float:
    files = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    return max(os.path.getmtime(f) for f in files)


def _compile(src: str, verbose: bool, build_dir: str = BUILD, defines=()) -> str:
    obj = os.path.join(build_dir, os.path.basename(src) + ".o")
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *[f"-D{d}" for d in defines], "-c", src, "-o", obj]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
    if verbose and r.stderr:
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Build libmoefp8.so (or, with debug=True, libmoefp8_debug.so) and return its path."""
    build_dir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug else (BUILD, LIB)
    defines = ("MOE_FAULT_INJECTION",) if debug else ()
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    dep = _deps_mtime()
    todo = []
    for s in srcs:
        obj = os.path.join(build_dir, os.path.basename(s) + ".o")
        if force or verbose or not os.path.exists(obj) or os.path.getmtime(obj) < max(dep, os.path.getmtime(s)):
            todo.append(s)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        list(ex.map(lambda s: _compile(s, verbose, build_dir, defines), todo))
    objs = [os.path.join(build_dir, os.path.basename(s) + ".o") for s in srcs]
    if todo or not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
        tmp = lib + f".{os.getpid()}.tmp"
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc link failed:\n{r.stderr}")
        os.replace(tmp, lib)
    return lib


def build_all(force: bool = False, verbose: bool = False) -> list:
    """The release library and the fault-injection debug library."""
    return [build(force, verbose), build(force, False, debug=True)]


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/spill usage")
    ap.add_argument("--debug", action="store_true", help="also build libmoefp8_debug.so")
    a = ap.parse_args()
    print(build_all(a.force, a.verbose) if a.debug else build(force=a.force, verbose=a.verbose))
