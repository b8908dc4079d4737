"""Builds libkvc.so in-tree with nvcc for sm_100a, and on request the range-checking
variant libkvc_checks.so (the same sources compiled with -DKVC_CHECKS=1).

Usage: python -m long_context_kv_kvc_b200.build [--force] [--jobs N] [--checks]
"""
from __future__ import annotations

import argparse
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libkvc.so")
OBJ_CHECKS = os.path.join(PKG, "_build_checks")
LIB_CHECKS = os.path.join(PKG, "libkvc_checks.so")

SOURCES = ["api.cu", "score_simt.cu", "score_tc.cu", "select.cu", "gather.cu", "noalloc.cu", "csm.cu", "decode.cu"]
HEADERS = ["kvc_internal.cuh", "tc_ptx.cuh"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE,
         "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, jobs: int = 8, verbose: bool = False, extra=(), checks: bool = False) -> str:
    obj_dir, lib = (OBJ_CHECKS, LIB_CHECKS) if checks else (OBJ, LIB)
    if checks:
        extra = (*extra, "-DKVC_CHECKS=1")
    os.makedirs(obj_dir, exist_ok=True)
    headers = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "kvc.h")]
    objs, todo = [], []
    for s in SOURCES:
        src = os.path.join(CSRC, s)
        obj = os.path.join(obj_dir, s.replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, [src] + headers + [__file__]):
            todo.append([NVCC, *FLAGS, *extra, "-c", src, "-o", obj])

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)

    with ThreadPoolExecutor(max(1, jobs)) as ex:
        list(ex.map(run, todo))
    if force or todo or _stale(lib, objs):
        run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", lib, *objs,
             "-Xcompiler", "-fPIC", "-cudart", "static"])
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=8)
    ap.add_argument("--ptxas-v", action="store_true", help="print register/smem usage")
    ap.add_argument("--checks", action="store_true", help="build libkvc_checks.so (KVC_CHECKS=1)")
    a = ap.parse_args()
    print(build(force=a.force or a.ptxas_v, jobs=a.jobs, verbose=True,
                extra=("-Xptxas", "-v") if a.ptxas_v else (), checks=a.checks))
