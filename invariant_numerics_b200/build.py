"""Build libinvnum.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m invariant_numerics_b200.build [--verbose] [--ptxas-info] [--debug-bounds]

Each .cu under csrc/ is compiled in parallel to an object in _build/, then
linked into invariant_numerics_b200/libinvnum.so (CUDA runtime linked
statically; the driver API is reached through the runtime's entry-point
query, so no libcuda link is needed).  --debug-bounds builds the
index-checking variant (-DINV_DEBUG_BOUNDS, objects in _build_debug/) as
invariant_numerics_b200/libinvnum_debug.so; the binding loads it instead of
libinvnum.so when the environment variable INVNUM_LIBRARY names it.
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
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libinvnum.so")
BUILD_DEBUG = os.path.join(ROOT, "_build_debug")
LIB_DEBUG = os.path.join(PKG, "libinvnum_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-I" + INCLUDE, "-I" + CSRC]


def nvcc() -> str:
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; set NVCC")
    return cand


def _compile(src: str, obj: str, extra, verbose: bool) -> str:
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return (r.stdout + r.stderr).strip()


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib) -> bool:
    if not os.path.exists(lib):
        return True
    lib_t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > lib_t for d in deps)


def build(verbose: bool = False, ptxas_info: bool = False, force: bool = False, debug_bounds: bool = False) -> str:
    """Compile (if stale) and return the path of libinvnum.so (of
    libinvnum_debug.so with debug_bounds)."""
    bdir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug_bounds else (BUILD, LIB)
    os.makedirs(bdir, exist_ok=True)
    srcs = sources()
    objs = [os.path.join(bdir, os.path.basename(s)[:-3] + ".o") for s in srcs]
    if not force and not ptxas_info and not _stale(lib):
        return lib
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    if debug_bounds:
        extra.append("-DINV_DEBUG_BOUNDS")
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        outs = list(ex.map(lambda so: _compile(so[0], so[1], extra, verbose), zip(srcs, objs)))
    if ptxas_info:
        for s, o in zip(srcs, outs):
            print(f"== {os.path.basename(s)}\n{o}")
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true", help="build libinvnum_debug.so (index checks)")
    a = ap.parse_args(argv)
    print(build(verbose=a.verbose, ptxas_info=a.ptxas_info, force=a.force, debug_bounds=a.debug_bounds))
    return 0


if __name__ == "__main__":
    sys.exit(main())
