"""Build the sm_100a CUDA library in-tree: block_sparse_attention_cube_b200/libvsa_b200.so.

Each .cu file under csrc/ is compiled by nvcc for sm_100a only
(``-gencode arch=compute_100a,code=sm_100a -lineinfo``) into _build/, then the
objects are linked into one shared library with the CUDA runtime linked
statically, so the library loads on a host without a GPU driver (its entry
points then return VSA_ERR_CUDA) and needs nothing beyond libc at load time.

Usage: ``python block_sparse_attention_cube_b200/build_lib.py [--force] [--ptxas-v]`` (run it as a
file: importing the package loads the library this script builds).
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
LIB = os.path.join(PKG, "libvsa_b200.so")

SOURCES = sorted(f for f in os.listdir(CSRC) if f.endswith(".cu"))
HEADERS = ["ptx_sm100.cuh", "vsa_internal.h"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or install CUDA 12.8+)")


def _newest_dep() -> float:
    deps = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "vsa.h"), os.path.abspath(__file__)]
    return max(os.path.getmtime(p) for p in deps)


def _compile(nvcc: str, src: str, obj: str, ptxas_v: bool) -> str:
    cmd = [nvcc, *ARCH, *CFLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
    if ptxas_v:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    return r.stderr


def build(force: bool = False, ptxas_v: bool = False, verbose: bool = False) -> str:
    """Compile (if stale) and link the library; return its path."""
    nvcc = nvcc_path()
    os.makedirs(BUILD, exist_ok=True)
    dep_time = _newest_dep()
    jobs = []
    objs = []
    for src in SOURCES:
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(obj)
        stale = force or ptxas_v or not os.path.exists(obj) or \
            os.path.getmtime(obj) < max(os.path.getmtime(os.path.join(CSRC, src)), dep_time)
        if stale:
            jobs.append((src, obj))
    logs = []
    if jobs:
        with cf.ThreadPoolExecutor(max_workers=len(jobs)) as ex:
            futs = {ex.submit(_compile, nvcc, s, o, ptxas_v): s for s, o in jobs}
            for f in cf.as_completed(futs):
                logs.append((futs[f], f.result()))
    if jobs or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        tmp = LIB + ".tmp"
        # every symbol must resolve inside the library (a source left out fails here, not at load time)
        cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-Xlinker", "--no-undefined", "-o", tmp, *objs,
               "-lpthread", "-ldl", "-lrt"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    if verbose or ptxas_v:
        for src, log in sorted(logs):
            if log.strip():
                print(f"--- {src}\n{log}", file=sys.stderr)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print register / shared-memory usage per kernel")
    a = ap.parse_args(argv)
    print(build(force=a.force, ptxas_v=a.ptxas_v, verbose=True))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
