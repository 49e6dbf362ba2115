"""Builds libsparse_attn.so in-tree with nvcc for sm_100a.

    python -m block_sparse_long_landmark_b200.build [--force] [--verbose] [--debug-bounds]

Each ``csrc/*.cu`` is compiled to an object under ``_build/`` (in parallel),
then linked into ``lib/libsparse_attn.so`` with the static CUDA runtime.
``--debug-bounds`` builds the address-checking variant (``-DSA_DEBUG_BOUNDS``:
every gather checks its first row against the slab it means to read and sets
status bit 8 when outside) under ``_build_bounds/`` into
``lib/libsparse_attn_bounds.so``.
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
BUILD_BOUNDS = os.path.join(PKG, "_build_bounds")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libsparse_attn.so")
LIB_BOUNDS = os.path.join(LIBDIR, "libsparse_attn_bounds.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
              "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _deps_mtime() -> float:
    files = glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return max(os.path.getmtime(f) for f in files)


def _compile(src: str, verbose: bool, extra: list[str], build_dir: str = BUILD) -> str:
    obj = os.path.join(build_dir, os.path.basename(src) + ".o")
    if os.path.exists(obj) and os.path.getmtime(obj) >= _deps_mtime():
        return obj
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, flush=True)
    return obj


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None, bounds: bool = False) -> str:
    """Compile (when sources are newer than the library) and return its path."""
    extra = list(extra or [])
    build_dir, lib = BUILD, LIB
    if bounds:
        build_dir, lib = BUILD_BOUNDS, LIB_BOUNDS
        extra.append("-DSA_DEBUG_BOUNDS")
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= _deps_mtime():
        return lib
    os.makedirs(build_dir, exist_ok=True)
    os.makedirs(LIBDIR, exist_ok=True)
    if force:
        for o in glob.glob(os.path.join(build_dir, "*.o")):
            os.remove(o)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    with ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, extra, build_dir), srcs))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", "-cudart", "static", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true", help="build the address-checking variant")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose, bounds=a.debug_bounds))


if __name__ == "__main__":
    sys.exit(main())
