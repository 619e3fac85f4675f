"""Build libmoe.so in-tree: nvcc for sm_100a, one object per source file.

    python -m mixture_experts_layer_33_b200.build [--force] [--verbose] [--debug]

Objects go to ``_build/`` at the repository root; the shared library lands
next to this file (``mixture_experts_layer_33_b200/libmoe.so``), where the
binding loads it from. ``--debug`` builds the MOE_DEBUG variant
(``libmoe_debug.so``, objects in ``_build/debug/``), whose kernels also
range-check the row offsets, rows and token lists callers hand in; the
binding loads it when the environment sets MOE_DEBUG=1.
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmoe.so")
BUILD_DEBUG = os.path.join(BUILD, "debug")
LIB_DEBUG = os.path.join(PKG, "libmoe_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
                     "-I", INCLUDE, "-I", CSRC]


def nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return hs


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, verbose, extra, build_dir=BUILD):
    obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
    cmd = [nvcc()] + NVCC_FLAGS + extra + ["-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(src)}:\n{r.stderr}")
    return obj, (r.stderr if verbose else "")


def build(force=False, verbose=False, extra_flags=(), debug=False):
    """Compile every CUDA source and link libmoe.so (libmoe_debug.so with
    ``debug``); returns its path."""
    build_dir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug else (BUILD, LIB)
    flags = list(extra_flags) + (["-DMOE_DEBUG=1"] if debug else [])
    os.makedirs(build_dir, exist_ok=True)
    srcs = sources()
    hdrs = headers()
    todo = [s for s in srcs
            if force or _stale(os.path.join(build_dir, os.path.basename(s)[:-3] + ".o"), [s] + hdrs)]
    logs = []
    if todo:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(todo))) as ex:
            for obj, log in ex.map(lambda s: _compile(s, verbose, flags, build_dir), todo):
                if log:
                    logs.append(log)
    objs = [os.path.join(build_dir, os.path.basename(s)[:-3] + ".o") for s in srcs]
    if force or todo or _stale(lib, objs):
        cmd = [nvcc()] + ARCH + ["-shared", "-o", lib] + objs + ["-cudart", "static"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr}")
    if verbose:
        sys.stdout.write("".join(logs))
    return lib


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print -Xptxas -v resource usage")
    ap.add_argument("--debug", action="store_true",
                    help="build the MOE_DEBUG variant (libmoe_debug.so)")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose, debug=a.debug))


if __name__ == "__main__":
    main()
