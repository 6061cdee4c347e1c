"""Builds libsma.so (the C-ABI library) in-tree for sm_100a with nvcc.

Usage: ``python -m structured_mask_attention_analytic_b200.csrc.build [--force] [-v]``
Objects go to ``_build/`` at the repository root; the library is written next
to the Python binding so that it travels with the source tree.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsma.so")

SOURCES = ["runtime.cu", "tile_maps.cu", "attn_tc.cu", "attn_simt.cu", "decode.cu", "topk.cu", "gather.cu", "tma_map.cu", "attn_bwd.cu", "attn_bwd_simt.cu", "varlen.cu",
           "noalloc.cu", "sma_api.cpp"]
HEADERS = ["device_common.cuh", "kernels.h", "gather.cuh", "tma_map.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", HERE,
         "--expt-relaxed-constexpr"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libsma")
    return path


def _newest_input(src: str) -> float:
    deps = [os.path.join(HERE, src)] + [os.path.join(HERE, h) for h in HEADERS]
    deps.append(os.path.join(INCLUDE, "sma.h"))
    return max(os.path.getmtime(d) for d in deps)


def _compile(src: str, force: bool, verbose: bool, extra: list[str]) -> str:
    obj = os.path.join(BUILD, src + ".o")
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= _newest_input(src):
        return obj
    cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-c", os.path.join(HERE, src), "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr, flush=True)
    return obj


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as pool:
        objs = list(pool.map(lambda s: _compile(s, force or ptxas_info, verbose or ptxas_info, extra),
                             SOURCES))
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        tmp = LIB + ".tmp"
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs, "-ldl", "-lrt",
               "-lpthread"]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
        os.replace(tmp, LIB)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers/spills per kernel")
    a = ap.parse_args(argv)
    print(build(a.force, a.verbose, a.ptxas_info))
    return 0


if __name__ == "__main__":
    sys.exit(main())
