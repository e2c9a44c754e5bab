"""Build libbi.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m invariant_deterministic_03_b200.build [--force] [--debug]

Each .cu file under csrc/ compiles to an object in csrc/_build/, then all are
linked into invariant_deterministic_03_b200/libbi.so against the shared CUDA
runtime (the same libcudart.so.12 that PyTorch loads).
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(CSRC, "_build")
LIB = os.path.join(HERE, "libbi.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
SOURCES = ["api.cu", "rmsnorm.cu", "gemm.cu", "attention.cu", "attention_noalloc.cu",
           "pointwise.cu", "upcast.cu", "forward.cu"]
HEADERS = ["common.cuh", "host.h"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xptxas", "-v"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps_mtime() -> float:
    files = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "bi.h"), __file__]
    return max(os.path.getmtime(f) for f in files)


def _compile(src: str, extra) -> tuple[str, str]:
    obj = os.path.join(BUILD, src.replace(".cu", ".o"))
    cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-I", INCLUDE, "-c", os.path.join(CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def build(force: bool = False, debug: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    extra = ["-DBI_DEBUG=1"] if debug else []
    dep = _deps_mtime()
    todo = []
    for src in SOURCES:
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(
                dep, os.path.getmtime(os.path.join(CSRC, src))):
            todo.append(src)
    with ThreadPoolExecutor(max_workers=min(8, len(SOURCES))) as ex:
        for obj, log in ex.map(lambda s: _compile(s, extra), todo):
            if verbose:
                sys.stdout.write(f"== {os.path.basename(obj)}\n{log}")
    objs = [os.path.join(BUILD, s.replace(".cu", ".o")) for s in SOURCES]
    if todo or not os.path.exists(LIB):
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "shared", "-o", LIB, *objs,
               "-Xlinker", "-rpath=/usr/local/cuda/lib64", "-Xlinker", "--no-undefined"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, debug=a.debug, verbose=a.verbose))
