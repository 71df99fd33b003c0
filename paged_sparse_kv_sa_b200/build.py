"""Build ``libsa.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m paged_sparse_kv_sa_b200.build [--jobs N] [--force]

Objects go to ``_build/`` at the repository root; the shared library lands
next to this file so that the Python binding finds it.
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
OBJ = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsa.so")
SOURCES = ["api.cu", "decode.cu", "prefill.cu", "mla.cu", "select.cu", "select_mla.cu", "combine.cu", "summaries.cu", "append.cu", "heads.cu",
           "union.cu"]
HEADERS = ["common.cuh", "exact.cuh", "tc05.cuh", "topk.cuh", "internal.h", os.path.join("..", "..", "include", "sa.h")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def _newest(paths):
    return max(os.path.getmtime(p) for p in paths if os.path.exists(p))


def _compile(src: str, force: bool, obj_dir: str = OBJ, defines=()) -> str:
    out = os.path.join(obj_dir, os.path.splitext(src)[0] + ".o")
    deps = [os.path.join(CSRC, src)] + [os.path.join(CSRC, h) for h in HEADERS]
    if not force and os.path.exists(out) and os.path.getmtime(out) >= _newest(deps):
        return out
    cmd = [nvcc(), *ARCH, *FLAGS, *[f"-D{d}" for d in defines], "-c", os.path.join(CSRC, src),
           "-o", out]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return out


def build(jobs: int = 0, force: bool = False, verbose: bool = False, defines=(), out: str = LIB,
          obj_dir: str = OBJ) -> str:
    """Compile every source and link ``out``; ``defines`` are extra -D macros
    (build-time kernel shapes, e.g. SA_DECODE_WARPS=4)."""
    os.makedirs(obj_dir, exist_ok=True)
    jobs = jobs or min(len(SOURCES), os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(jobs) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, obj_dir, defines), SOURCES))
    if force or not os.path.exists(out) or os.path.getmtime(out) < _newest(objs):
        cmd = [nvcc(), *ARCH, "-shared", "-o", out, *objs, "-lcudart"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    if verbose:
        print(out)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--jobs", type=int, default=0)
    ap.add_argument("--force", action="store_true")
    args = ap.parse_args()
    build(args.jobs, args.force, verbose=True)
    sys.exit(0)
