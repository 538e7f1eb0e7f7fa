"""Build libdsa.so (the C-ABI CUDA library) in-tree for sm_100a.

Usage: ``python -m sparse_attention_sum_b200.build [--jobs N] [--force]``.
Each ``csrc/*.cu`` file compiles to an object under ``_build/`` and the
objects link into ``sparse_attention_sum_b200/libdsa.so``.  A file is rebuilt
when it or any header under ``csrc/`` or ``include/`` is newer than its object.
Each source's compiler output (ptxas register and spill report, warnings) is
kept in ``_build/<name>.log`` and ``_build/ptxas.log`` is their concatenation
for the current objects.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libdsa.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
              "-Xptxas", "-v", "-I", INCLUDE, "-I", CSRC] + ARCH


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _compile(src: str, obj: str) -> tuple:
    cmd = [nvcc(), "-c", src, "-o", obj] + NVCC_FLAGS
    p = subprocess.run(cmd, capture_output=True, text=True)
    return src, p.returncode, p.stdout + p.stderr


def build(jobs: int = 8, force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr_mtime = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    todo = []
    objs = []
    for s in srcs:
        o = os.path.join(BUILD, os.path.basename(s)[:-3] + ".o")
        objs.append(o)
        if force or not os.path.exists(o) or os.path.getmtime(o) < max(os.path.getmtime(s), hdr_mtime):
            todo.append((s, o))
    if todo:
        with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
            for src, rc, out in ex.map(lambda so: _compile(*so), todo):
                with open(os.path.join(BUILD, os.path.basename(src)[:-3] + ".log"), "w") as f:
                    f.write(out)
                if rc != 0:
                    raise RuntimeError(f"nvcc failed for {os.path.basename(src)}:\n{out}")
                if verbose:
                    print(f"== {os.path.basename(src)}\n{out}")
    need_link = bool(todo) or not os.path.exists(LIB) or \
        os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs)
    if need_link:
        tmp = LIB + ".tmp"
        cmd = [nvcc(), "-shared", "-o", tmp] + objs + ARCH + ["-cudart", "shared",
                                                              "-Xlinker", "-rpath,/usr/local/cuda/lib64"]
        p = subprocess.run(cmd, capture_output=True, text=True)
        if p.returncode != 0:
            raise RuntimeError(f"link failed:\n{p.stdout}{p.stderr}")
        os.replace(tmp, LIB)
    with open(os.path.join(BUILD, "ptxas.log"), "w") as f:
        for s in srcs:
            log = os.path.join(BUILD, os.path.basename(s)[:-3] + ".log")
            if os.path.exists(log):
                f.write(f"== {os.path.basename(s)}\n" + open(log).read())
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--jobs", type=int, default=os.cpu_count() or 4)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build(a.jobs, a.force, a.verbose))


if __name__ == "__main__":
    sys.exit(main())
