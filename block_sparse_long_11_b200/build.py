"""Build libmoba.so in-tree with nvcc for sm_100a (B200).

    python -m block_sparse_long_11_b200.build [--verbose] [--ptxas-info] [--debug]

Each csrc/*.cu is compiled to an object under _build/ (skipped when the
object is newer than every source and header), then linked into
block_sparse_long_11_b200/libmoba.so.  The CUDA runtime is linked statically.
--debug builds the bounds-checked variant instead: -DMOBA_DEBUG, objects
under _build/debug/, block_sparse_long_11_b200/libmoba_debug.so (loaded when
MOBA_DEBUG=1 is set in the environment).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmoba.so")
BUILD_DEBUG = os.path.join(BUILD, "debug")
LIB_DEBUG = os.path.join(PKG, "libmoba_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _flags(ptxas_info: bool, debug: bool = False):
    f = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC]
    if debug:
        f += ["-DMOBA_DEBUG=1"]
    if ptxas_info:
        f += ["-Xptxas", "-v"]
    return f


def build(verbose: bool = False, ptxas_info: bool = False, force: bool = False,
          debug: bool = False) -> str:
    BUILD_DIR = BUILD_DEBUG if debug else BUILD
    OUT = LIB_DEBUG if debug else LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))
    newest_header = max([os.path.getmtime(h) for h in headers] + [0])
    objs, jobs = [], []
    for src in sources:
        obj = os.path.join(BUILD_DIR, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if (not force and not ptxas_info and os.path.exists(obj)
                and os.path.getmtime(obj) > max(os.path.getmtime(src), newest_header)):
            continue
        jobs.append((src, [nvcc()] + _flags(ptxas_info, debug) + ["-c", src, "-o", obj]))
    # one nvcc per out-of-date source, run side by side; outputs in source order
    with ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        results = list(ex.map(lambda j: subprocess.run(j[1], capture_output=True, text=True), jobs))
    for (src, cmd), r in zip(jobs, results):
        if verbose:
            print(" ".join(cmd), flush=True)
        if r.returncode != 0 or verbose or ptxas_info:
            sys.stderr.write(r.stdout + r.stderr)
    for (src, _), r in zip(jobs, results):
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}")
    if (force or not os.path.exists(OUT)
            or os.path.getmtime(OUT) < max(os.path.getmtime(o) for o in objs)):
        tmp = OUT + ".tmp"
        cmd = [nvcc()] + ARCH + ["-shared", "-o", tmp] + objs
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"link of {os.path.basename(OUT)} failed")
        os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, ptxas_info="--ptxas-info" in sys.argv,
                force="--force" in sys.argv, debug="--debug" in sys.argv))
