"""Build libfa.so in-tree with nvcc for sm_100a.

    python -m exact_io_aware_80_b200.build [--force] [--jobs N] [--checks]

Each .cu file under csrc/ is compiled to an object in csrc/_build/ (skipped
when the object is newer than every source and header), then all objects are
linked into exact_io_aware_80_b200/libfa.so.  --checks builds the same ABI with
device-side index checks (FA_CHECKS) into csrc/_build_checks/ and
libfa_checks.so.  No GPU is needed: nvcc cross-compiles.
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
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(CSRC, "_build")
BUILD_CHECKS = os.path.join(CSRC, "_build_checks")
LIB = os.path.join(PKG, "libfa.so")
LIB_CHECKS = os.path.join(PKG, "libfa_checks.so")
ROOT = os.path.dirname(PKG)

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC,-O2",
         "-I" + os.path.join(ROOT, "include"), "-I" + CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; set NVCC or put the CUDA toolkit on PATH")


def _newest_header() -> float:
    hs = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))
    return max((os.path.getmtime(h) for h in hs), default=0.0)


def _compile(src: str, force: bool, extra, build_dir: str = BUILD) -> str:
    obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(src), _newest_header()):
        return obj
    cmd = [nvcc()] + ARCH + FLAGS + list(extra) + os.environ.get("FA_NVCC_EXTRA", "").split() + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    if r.stderr.strip():
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, jobs: int = 0, extra=(), checks: bool = False) -> str:
    """Build libfa.so, or with checks=True libfa_checks.so: the same sources compiled with
    FA_CHECKS, whose kernels check their direct memory accesses against the tensors' sizes
    and record FA_ERR_BOUNDS in the device status word instead of making the access."""
    build_dir = BUILD_CHECKS if checks else BUILD
    lib = LIB_CHECKS if checks else LIB
    extra = list(extra) + (["-DFA_CHECKS"] if checks else [])
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    jobs = jobs or min(len(srcs), os.cpu_count() or 4)
    with cf.ThreadPoolExecutor(jobs) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, extra, build_dir), srcs))
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
        cmd = [nvcc()] + ARCH + ["-shared", "-o", lib] + objs + ["-lcudart"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=0)
    ap.add_argument("--ptxas-verbose", action="store_true", help="print register / spill / smem usage")
    ap.add_argument("--checks", action="store_true", help="build libfa_checks.so (device-side index checks)")
    a = ap.parse_args()
    extra = ["-Xptxas", "-v"] if a.ptxas_verbose else []
    print(build(force=a.force or a.ptxas_verbose, jobs=a.jobs, extra=extra, checks=a.checks))


if __name__ == "__main__":
    main()
