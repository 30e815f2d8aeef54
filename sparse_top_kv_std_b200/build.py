"""Build the C-ABI shared library ``libstd_b200.so`` for sm_100a (B200) in-tree.

    python -m sparse_top_kv_std_b200.build [--verbose] [--ptxas-info] [--product-only]

Each CUDA source is compiled to an object in ``_build/`` (in parallel), then
linked into ``sparse_top_kv_std_b200/libstd_b200.so``.  The same sources are also
compiled with -DSTD_DEBUG into ``_build/debug/`` and linked into
``libstd_b200_debug.so``: device-side bounds checks of every index and cache row
(STD_DEVERR_DEBUG), loaded instead of the product library when STD_B200_DEBUG=1.
nvcc cross-compiles, so this runs without a GPU.
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
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_NAME = "libstd_b200.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3", "--expt-relaxed-constexpr",
              "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; set NVCC or put the CUDA toolkit on PATH")
    return cand


def _newer(out: str, deps) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(d) <= t for d in deps)


DEBUG_LIB_PATH = os.path.join(PKG, "libstd_b200_debug.so")


def build(verbose: bool = False, ptxas_info: bool = False, force: bool = False, debug: bool = None) -> str:
    """Compile every ``csrc/*.cu`` for sm_100a and link ``libstd_b200.so``; return its path.

    debug=True builds ``libstd_b200_debug.so`` instead: the same sources with -DSTD_DEBUG
    (device-side bounds checks of every index and cache row, reported as STD_DEVERR_DEBUG).
    debug=None (the default) builds both, the product library last."""
    if debug is None:
        build(verbose, False, force, debug=True)
        return build(verbose, ptxas_info, force, debug=False)
    build_dir = os.path.join(BUILD_DIR, "debug") if debug else BUILD_DIR
    lib_path = DEBUG_LIB_PATH if debug else LIB_PATH
    os.makedirs(build_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                     + glob.glob(os.path.join(ROOT, "include", "*.h")))
    extra = (["-Xptxas", "-v"] if ptxas_info else []) + (["-DSTD_DEBUG"] if debug else [])

    def compile_one(src: str) -> str:
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        if not force and not ptxas_info and _newer(obj, [src, __file__] + headers):
            return obj
        cmd = [nvcc()] + ARCH + NVCC_FLAGS + extra + ["-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if (verbose or ptxas_info) and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, flush=True)
        return obj

    with ThreadPoolExecutor(min(8, len(sources))) as ex:
        objs = list(ex.map(compile_one, sources))
    if force or ptxas_info or not _newer(lib_path, objs):
        cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", lib_path] + objs
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib_path


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills / smem per kernel")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--product-only", action="store_true", help="skip the debug build (libstd_b200_debug.so)")
    args = ap.parse_args(argv)
    path = build(verbose=args.verbose, ptxas_info=args.ptxas_info, force=args.force,
                 debug=False if args.product_only else None)
    print(path)
    return 0


if __name__ == "__main__":
    sys.exit(main())
