"""Build libgdr.so in-tree for sm_100a with nvcc.

    python gated_delta_rule_forward_b200/csrc/build.py [--force] [-j N]

Each .cu file under csrc/ is compiled to an object in
gated_delta_rule_forward_b200/_build/ (ptxas register/spill reports go to
_build/ptxas.log), and the objects are linked with the static CUDA runtime
into gated_delta_rule_forward_b200/libgdr.so.  Objects are rebuilt when their
source or any header is newer.  No GPU is needed to build.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

CSRC = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(CSRC)
ROOT = os.path.dirname(PKG)
BUILD = os.path.join(PKG, "_build")
OUT = os.path.join(PKG, "libgdr.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
          "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-Xptxas", "-v"]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, force):
    obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
    log = obj + ".ptxas.txt"
    if not force and not _stale(obj, [src] + _headers()):
        return obj, None
    cmd = [NVCC] + ARCH + CFLAGS + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    with open(log, "w") as f:
        f.write(r.stdout + r.stderr)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stderr[-6000:]}")
    return obj, log


def build(force: bool = False, jobs: int = 8, verbose: bool = True) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        results = list(ex.map(lambda s: _compile(s, force), srcs))
    objs = [o for o, _ in results]
    if force or _stale(OUT, objs):
        tmp = OUT + f".tmp{os.getpid()}"
        cmd = [NVCC] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr[-4000:]}")
        os.replace(tmp, OUT)
        if verbose:
            print(f"built {OUT}")
    with open(os.path.join(BUILD, "ptxas.log"), "w") as f:
        for src in srcs:
            p = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o.ptxas.txt")
            if os.path.exists(p):
                f.write(f"==== {os.path.basename(src)}\n" + open(p).read())
    return OUT


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=8)
    a = ap.parse_args()
    try:
        build(force=a.force, jobs=a.j)
    except RuntimeError as e:
        print(e, file=sys.stderr)
        sys.exit(1)
