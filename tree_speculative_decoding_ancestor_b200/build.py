"""Build libtsd.so in-tree with nvcc for sm_100a.

    python -m tree_speculative_decoding_ancestor_b200.build [--force] [--verbose]

Objects go to ``_build/`` next to this file, the library to ``lib/libtsd.so``.
nvcc cross-compiles for sm_100a without a GPU.
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import subprocess
import sys
from typing import List

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB_DIR = os.path.join(HERE, "lib")
LIB = os.path.join(LIB_DIR, "libtsd.so")
# The checked build (-DTSD_CHECKS): every global access whose index a kernel
# computes is compared with its buffer's extent first; an index outside it
# sets TSD_DEV_BOUNDS in the status word and the access is skipped.  Slower;
# for small-case debugging.  Load it with TSD_LIBRARY=<path> before the
# binding's first call.
LIB_CHECKED = os.path.join(LIB_DIR, "libtsd_checked.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
          "--expt-relaxed-constexpr", "-Xcompiler", "-Wall"]


def _sources() -> List[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _headers() -> List[str]:
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return hs


def _stale(target: str, deps: List[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, force: bool, verbose: bool, checked: bool = False) -> str:
    obj = os.path.join(BUILD, os.path.basename(src)[:-3] + (".checked.o" if checked else ".o"))
    if force or _stale(obj, [src] + _headers()):
        cmd = [NVCC] + ARCH + CFLAGS + (["-DTSD_CHECKS"] if checked else []) + \
            (["-Xptxas", "-v"] if verbose else []) + ["-c", src, "-o", obj + ".tmp"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and r.stderr:
            sys.stderr.write(r.stderr)
        os.replace(obj + ".tmp", obj)
    return obj


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Compile every source and link the library (the checked build with
    `checked`); returns its path."""
    os.makedirs(BUILD, exist_ok=True)
    os.makedirs(LIB_DIR, exist_ok=True)
    srcs = _sources()
    lib = LIB_CHECKED if checked else LIB
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, verbose, checked), srcs))
    if force or _stale(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [NVCC] + ARCH + ["-shared", "-o", tmp] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--checked", action="store_true", help="the bounds-checked debug build")
    args = ap.parse_args()
    print(build(args.force, args.verbose, args.checked))
