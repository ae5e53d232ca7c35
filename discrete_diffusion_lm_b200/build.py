"""Build libdg.so (sm_100a) in-tree with nvcc.

    python -m discrete_diffusion_lm_b200.build [--force] [--verbose] [--checks]

With --checks the same sources are compiled with DG_CHECKS=1 into libdg_checks.so (objects under
_build/checks/): the kernels then verify their index invariants and the token ids they are given,
record code 2 in their device error word on a violation and skip the access (see
include/dg.h, dg_device_error).

Every translation unit is compiled for sm_100a only
(-gencode arch=compute_100a,code=sm_100a) with line info, and linked into
discrete_diffusion_lm_b200/libdg.so against the static CUDA runtime.  Object
files go to _build/ at the repository root.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libdg.so")
LIB_CHECKS = os.path.join(PKG, "libdg_checks.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-ffp-contract=off",
                 "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _headers():
    return (glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, verbose: bool, out_dir: str = BUILD, extra=()) -> str:
    obj = os.path.join(out_dir, os.path.basename(src) + ".o")
    cmd = [NVCC] + COMMON + list(extra) + ["-c", src, "-o", obj]
    if verbose and src.endswith(".cu"):
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        sys.stdout.write(r.stdout + r.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, checks: bool = False) -> str:
    """Compile and link libdg.so (libdg_checks.so with `checks`) if any source or header is newer;
    return its path."""
    out_dir = os.path.join(BUILD, "checks") if checks else BUILD
    lib = LIB_CHECKS if checks else LIB
    extra = ["-DDG_CHECKS=1"] if checks else []
    os.makedirs(out_dir, exist_ok=True)
    srcs = _sources()
    hdrs = _headers()
    todo = [s for s in srcs if force or _stale(os.path.join(out_dir, os.path.basename(s) + ".o"), [s] + hdrs)]
    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(todo)))) as ex:
        list(ex.map(lambda s: _compile(s, verbose, out_dir, extra), todo))
    objs = [os.path.join(out_dir, os.path.basename(s) + ".o") for s in srcs]
    if force or todo or _stale(lib, objs):
        cmd = [NVCC] + ARCH + ["-shared", "-cudart", "static", "-o", lib] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--checks", action="store_true", help="build libdg_checks.so (DG_CHECKS=1)")
    a = ap.parse_args()
    print(build(a.force, a.verbose, a.checks))
