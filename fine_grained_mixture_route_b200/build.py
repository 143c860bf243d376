"""Build the sm_100a shared library `libmoe_b200.so` in-tree with nvcc.

    python -m fine_grained_mixture_route_b200.build [--debug] [-j N]

Each .cu under csrc/ compiles to an object in _build/ (in parallel, skipped when up to
date), then nvcc links them into fine_grained_mixture_route_b200/libmoe_b200.so.  Only the
moe_* C entry points are exported.
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
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmoe_b200.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(debug: bool):
    f = ARCH + ["-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                "-I", os.path.join(ROOT, "include"), "--expt-relaxed-constexpr"]
    f += ["-O0", "-G"] if debug else ["-O3"]
    return f


def _needs(obj: str, deps) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in deps)


def build(debug: bool = False, jobs: int = 8, verbose: bool = False, ptxas_info: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))
    cc = nvcc()
    objs, cmds = [], []
    for s in srcs:
        o = os.path.join(BUILD, os.path.basename(s) + (".dbg.o" if debug else ".o"))
        objs.append(o)
        if _needs(o, [s] + headers + [__file__]) or ptxas_info:
            cmd = [cc] + flags(debug) + (["-Xptxas", "-v"] if ptxas_info else []) + ["-c", s, "-o", o]
            cmds.append(cmd)

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    failed = False
    with cf.ThreadPoolExecutor(max_workers=max(1, jobs)) as ex:
        for cmd, r in ex.map(run, cmds):
            if r.returncode != 0 or ptxas_info:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode != 0:
                failed = True
    if failed:
        raise RuntimeError("nvcc compilation failed")
    if _needs(LIB, objs):
        cmd = [cc] + ARCH + ["-shared", "-o", LIB] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("link failed")
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--debug", action="store_true")
    ap.add_argument("-j", type=int, default=8)
    ap.add_argument("-v", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills / shared memory per kernel")
    a = ap.parse_args()
    print(build(a.debug, a.j, a.v, a.ptxas_info))


if __name__ == "__main__":
    main()
