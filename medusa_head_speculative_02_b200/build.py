"""Builds libmedusa.so (all CUDA sources, sm_100a) in-tree with nvcc, and
libmedusa_debug.so, the same sources compiled with MEDUSA_DEBUG (device
index checks that report MEDUSA_ERR_BOUNDS instead of reading out of range).

Usage: python -m medusa_head_speculative_02_b200.build [--force] [--jobs N]
                                                      [--debug-only | --no-debug]
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
LIB = os.path.join(PKG, "libmedusa.so")
LIB_DEBUG = os.path.join(PKG, "libmedusa_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-rdc=true", "-Xcompiler", "-fPIC",
                     "-Xcompiler", "-Wall", "--expt-relaxed-constexpr", "-I", INCLUDE,
                     "-I", CSRC]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def headers() -> list[str]:
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return hs


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, obj: str, extra: list[str]) -> None:
    cmd = [nvcc()] + NVCC_FLAGS + extra + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(src)}:\n{r.stderr}")
    if r.stderr.strip():
        sys.stderr.write(r.stderr)


def build(force: bool = False, jobs: int = 0, verbose_ptxas: bool = False,
          debug: bool = False) -> str:
    """Compiles the release (debug=False) or MEDUSA_DEBUG library; returns its path."""
    bdir = os.path.join(BUILD, "debug") if debug else BUILD
    lib = LIB_DEBUG if debug else LIB
    os.makedirs(bdir, exist_ok=True)
    hdrs = headers()
    objs, todo = [], []
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    if debug:
        extra = extra + ["-DMEDUSA_DEBUG"]
    for src in sources():
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or verbose_ptxas or _stale(obj, [src] + hdrs):
            todo.append((src, obj))
    jobs = jobs or min(8, os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        list(ex.map(lambda so: _compile(so[0], so[1], extra), todo))
    if todo or _stale(lib, objs):
        cmd = [nvcc()] + ARCH + ["-shared", "-rdc=true", "-Xcompiler", "-fPIC", "-o", lib] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr}")
    return lib


def build_all(force: bool = False, jobs: int = 0) -> list[str]:
    """Both libraries (release and MEDUSA_DEBUG)."""
    return [build(force, jobs), build(force, jobs, debug=True)]


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=0)
    ap.add_argument("--ptxas-v", action="store_true", help="print register/smem usage")
    ap.add_argument("--debug-only", action="store_true", help="only libmedusa_debug.so")
    ap.add_argument("--no-debug", action="store_true", help="only libmedusa.so")
    a = ap.parse_args()
    if not a.debug_only:
        print(build(a.force, a.jobs, a.ptxas_v))
    if not a.no_debug:
        print(build(a.force, a.jobs, a.ptxas_v, debug=True))
