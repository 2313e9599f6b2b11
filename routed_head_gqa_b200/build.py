"""Build libgqe.so (and the test-only libgqe_selftest.so) in-tree with nvcc for sm_100a.

    python -m routed_head_gqa_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libgqe.so")
SELFTEST_LIB = os.path.join(PKG, "libgqe_selftest.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", os.path.join(os.path.dirname(PKG), "include")]

LIB_SOURCES = ["gqe_api.cu", "router.cu", "router_tc.cu", "prefill_simt.cu", "prefill_tc.cu", "decode.cu",
               "output.cu", "qproj.cu", "proj_tc.cu", "backward.cu", "backward_tc.cu", "route_bwd.cu", "aux_loss.cu"]
SELFTEST_SOURCES = ["selftest.cu"]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(os.path.dirname(PKG), "include", "gqe.h")]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, verbose):
    obj = os.path.join(BUILD, os.path.basename(src).replace(".cu", ".o"))
    if _stale(obj, [src] + _headers()):
        cmd = [NVCC, *ARCH, *FLAGS, "-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{res.stderr}")
        if verbose and res.stderr:
            print(res.stderr, file=sys.stderr)
    return obj


def _link(objs, out):
    tmp = out + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static", "-ldl", "-lpthread", "-lrt"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed for {out}:\n{res.stderr}")
    os.replace(tmp, out)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    if force:
        for f in glob.glob(os.path.join(BUILD, "*.o")):
            os.remove(f)
    for sources, out in ((LIB_SOURCES, LIB), (SELFTEST_SOURCES, SELFTEST_LIB)):
        srcs = [os.path.join(CSRC, s) for s in sources]
        with concurrent.futures.ThreadPoolExecutor(max_workers=len(srcs)) as ex:
            objs = list(ex.map(lambda s: _compile(s, verbose), srcs))
        if force or _stale(out, objs):
            _link(objs, out)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
