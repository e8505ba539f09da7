"""Build libbased.so in-tree for sm_100a with nvcc (no GPU needed to compile).

    python -m linear_attention_sequence_causal_b200.build [--force] [--verbose] [--debug-bounds]

Each csrc/*.cu compiles to an object under _build/ (skipped when newer than its
sources), then everything links into linear_attention_sequence_causal_b200/libbased.so
with the CUDA runtime linked statically. --debug-bounds builds the debug
library libbased_debug.so instead (objects under _build/debug/), compiled with
BASED_DEBUG_BOUNDS: the kernels check the index of every hand-indexed global
store and report an index outside its buffer as BASED_ERR_BOUNDS rather than
writing there.
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
LIB = os.path.join(PKG, "libbased.so")
DEBUG_LIB = os.path.join(PKG, "libbased_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + [
    "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr", "-I" + INCLUDE, "-I" + CSRC,
]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libbased")
    return exe


def _deps() -> list[str]:
    return (glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target: str, sources: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def _compile(src: str, force: bool, verbose: bool, extra: list[str], build_dir: str = BUILD) -> str:
    obj = os.path.join(build_dir, os.path.basename(src).replace(".cu", ".o"))
    if force or _stale(obj, [src] + _deps()):
        cmd = [nvcc()] + NVCC_FLAGS + extra + ["-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and r.stderr.strip():
            print(r.stderr, flush=True)
    return obj


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False, debug_bounds: bool = False) -> str:
    build_dir = os.path.join(BUILD, "debug") if debug_bounds else BUILD
    lib = DEBUG_LIB if debug_bounds else LIB
    os.makedirs(build_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    extra = (["-Xptxas", "-v"] if ptxas_info else []) + (["-DBASED_DEBUG_BOUNDS"] if debug_bounds else [])
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, verbose, extra, build_dir), sources))
    if force or _stale(lib, objs):
        cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", lib] + objs
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib


def main(argv=None) -> int:
    p = argparse.ArgumentParser(description=__doc__)
    p.add_argument("--force", action="store_true")
    p.add_argument("--verbose", action="store_true")
    p.add_argument("--ptxas-info", action="store_true", help="print register/smem use (-Xptxas -v)")
    p.add_argument("--debug-bounds", action="store_true", help="build the index-checking debug library")
    args = p.parse_args(argv)
    print(build(args.force, args.verbose or args.ptxas_info, args.ptxas_info, args.debug_bounds))
    return 0


if __name__ == "__main__":
    sys.exit(main())
