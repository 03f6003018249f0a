"""Builds libhq.so (sm_100a) in-tree with nvcc, and its bounds-checking build libhq_bounds.so
(the same sources with HQ_DEBUG_BOUNDS and relocatable device code, for the device word the
index checks share).

    python post_weight_quantization_tcgen05_b200/build.py [--force] [--bounds | --all]

(Run it as a script, or load it by path: importing it through the package would first import
the binding, which needs the library this script builds.)

The library is written next to this file so that it travels with the repository checkout.
Rebuilds only when a source under csrc/ or include/ is newer than the library.
"""

from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libhq.so")
LIB_BOUNDS = os.path.join(PKG, "libhq_bounds.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
]
OBJ_DIR = os.path.join(ROOT, "_build")


def _nvcc() -> str:
    for cand in (os.environ.get("CUDA_HOME", ""), "/usr/local/cuda"):
        p = os.path.join(cand, "bin", "nvcc") if cand else ""
        if p and os.path.exists(p):
            return p
    return "nvcc"


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd: list[str], verbose: bool) -> None:
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, cwd=PKG, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libhq.so")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)


def build(force: bool = False, verbose: bool = False, bounds: bool = False) -> str:
    """Compiles every translation unit to an object (in parallel), then links the library
    (libhq.so, or libhq_bounds.so with `bounds`)."""
    lib = LIB_BOUNDS if bounds else LIB
    if not force and not _stale(lib):
        return lib
    from concurrent.futures import ThreadPoolExecutor
    obj_dir = os.path.join(OBJ_DIR, "bounds") if bounds else OBJ_DIR
    extra = ["-DHQ_DEBUG_BOUNDS", "-rdc=true"] if bounds else []
    os.makedirs(obj_dir, exist_ok=True)
    objs = [os.path.join(obj_dir, os.path.basename(src)[:-3] + ".o") for src in sources()]
    cmds = [[_nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-c", "-o", obj, src] for src, obj in zip(sources(), objs)]
    with ThreadPoolExecutor(max_workers=max(1, min(len(cmds), os.cpu_count() or 1))) as ex:
        for f in [ex.submit(_run, c, verbose) for c in cmds]:
            f.result()
    tmp = lib + ".tmp"
    link = [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared"]
    if bounds:
        link.append("-rdc=true")
    _run([*link, "-o", tmp, *objs], verbose)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--bounds", action="store_true", help="build libhq_bounds.so only")
    ap.add_argument("--all", action="store_true", help="build libhq.so and libhq_bounds.so")
    args = ap.parse_args()
    if args.bounds or args.all:
        print(build(force=args.force, verbose=args.verbose, bounds=True))
    if not args.bounds:
        print(build(force=args.force, verbose=args.verbose))
