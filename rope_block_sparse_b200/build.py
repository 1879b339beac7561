"""Build libh3a.so in-tree for sm_100a with nvcc.

    python -m rope_block_sparse_b200.build [--force] [--verbose]

Each .cu file is compiled to an object under ``_build/`` (in parallel), then
linked into ``rope_block_sparse_b200/libh3a.so`` with the CUDA runtime linked
statically, so the library loads on a machine without a GPU driver (calls
that reach CUDA then fail with H3A_ERR_CUDA).  ``ptxas -v`` output (registers,
spills, shared memory) is kept in ``_build/<name>.ptxas.txt``.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libh3a.so")
SOURCES = ["h3a_api.cu", "prologue.cu", "router.cu", "attention.cu", "selftest.cu", "route_noalloc.cu", "dit_ops.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-Xptxas", "-v", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libh3a")


def _inputs() -> list:
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "h3a.h"))
    return files


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    nvcc = _nvcc()
    os.makedirs(BUILD, exist_ok=True)
    procs = []
    for src in SOURCES:
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        cmd = [nvcc, *ARCH, *FLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
        log = open(os.path.join(BUILD, src.replace(".cu", ".ptxas.txt")), "w")
        procs.append((src, obj, subprocess.Popen(cmd, stdout=log, stderr=subprocess.STDOUT), log))
    failed = []
    for src, obj, p, log in procs:
        p.wait()
        log.close()
        if p.returncode != 0:
            failed.append(src)
        if verbose or p.returncode != 0:
            sys.stderr.write(open(log.name).read())
    if failed:
        raise RuntimeError(f"nvcc failed on {failed}")
    tmp = LIB + f".tmp{os.getpid()}"
    link = [nvcc, *ARCH, "-shared", "-o", tmp, *[o for _, o, _, _ in procs], "-cudart", "static"]
    subprocess.check_call(link)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose))
