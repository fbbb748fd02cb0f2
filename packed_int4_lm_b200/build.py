"""Build libarchead.so in-tree with nvcc for sm_100a (B200).

    python -m packed_int4_lm_b200.build [--force] [--jobs N]

Each .cu under csrc/ compiles to an object under _build/ (rebuilt when it or a header
is newer), then one shared library is linked next to this file.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libarchead.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


TESTHOOKS_LIB = os.path.join(HERE, "libarchead_testhooks.so")


def _compile(src: str, force: bool, extra, outdir: str = BUILD) -> str:
    obj = os.path.join(outdir, os.path.basename(src)[:-3] + ".o")
    newest = max([os.path.getmtime(src)] + [os.path.getmtime(h) for h in _headers()])
    if force or not os.path.exists(obj) or os.path.getmtime(obj) < newest:
        cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        if r.stderr.strip():
            sys.stderr.write(r.stderr)
    return obj


def _link(lib: str, objs, force: bool) -> None:
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < max(map(os.path.getmtime, objs)):
        cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", lib, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")


def build(force: bool = False, jobs: int = 8, extra=(), testhooks: bool = True) -> str:
    """Build libarchead.so and, unless testhooks is False, the failure-detection test build
    libarchead_testhooks.so (the same sources with ARCHEAD_TEST_HOOKS defined)."""
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, list(extra)), srcs))
        _link(LIB, objs, force)
        if testhooks:
            tdir = os.path.join(BUILD, "testhooks")
            os.makedirs(tdir, exist_ok=True)
            tobjs = list(ex.map(lambda s: _compile(s, force, ["-DARCHEAD_TEST_HOOKS"], tdir), srcs))
            _link(TESTHOOKS_LIB, tobjs, force)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=8)
    ap.add_argument("--ptxas-v", action="store_true", help="print register/smem usage")
    a = ap.parse_args()
    print(build(a.force, a.jobs, ["-Xptxas", "-v"] if a.ptxas_v else []))
