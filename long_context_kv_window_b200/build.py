"""Build libkvc.so in-tree with nvcc for sm_100a.

    python -m long_context_kv_window_b200.build [--force] [--verbose]

Each .cu under csrc/ is compiled to an object in csrc/_build/ (in parallel)
and linked into long_context_kv_window_b200/libkvc.so with the CUDA runtime
linked statically.  Rebuilds only when a source or header is newer than the
library.

A second, test-only library libkvc_shortwait.so holds the scoring entry
points built with a pipeline-wait bound of a few nanoseconds
(KVC_WAIT_LIMIT_NS): its kernels give up their first wait, record
KVC_DEV_ERR_TIMEOUT and unwind, which is how the tests exercise the bounded
waits without a hang.  Nothing but the tests loads it.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(CSRC, "_build")
LIB = os.path.join(PKG, "libkvc.so")
SHORTWAIT_LIB = os.path.join(PKG, "libkvc_shortwait.so")
SHORTWAIT_SOURCES = ("score.cu", "api.cu")  # the entry points with pipeline waits, and what they need
SHORTWAIT_FLAGS = ["-DKVC_WAIT_LIMIT_NS=1ull"]
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
                 "--expt-relaxed-constexpr", "-Xcompiler", "-Wall"]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [
        os.path.abspath(__file__)]


def up_to_date() -> bool:
    if not os.path.exists(LIB) or not os.path.exists(SHORTWAIT_LIB):
        return False
    t = min(os.path.getmtime(LIB), os.path.getmtime(SHORTWAIT_LIB))
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    if not force and not ptxas_info and up_to_date():
        return LIB
    nvcc = _nvcc()
    os.makedirs(OBJ, exist_ok=True)
    srcs = _sources()
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    jobs = [(src, "", []) for src in srcs]
    jobs += [(os.path.join(CSRC, n), "_shortwait", SHORTWAIT_FLAGS) for n in SHORTWAIT_SOURCES]

    def compile_one(job) -> str:
        src, suffix, flags = job
        obj = os.path.join(OBJ, os.path.basename(src)[:-3] + suffix + ".o")
        cmd = [nvcc] + CFLAGS + flags + (extra if not suffix else []) + ["-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if (verbose or ptxas_info) and not suffix:
            print(r.stdout + r.stderr)
        return obj

    with ThreadPoolExecutor(max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(compile_one, jobs))
    for lib, lib_objs in ((LIB, objs[:len(srcs)]), (SHORTWAIT_LIB, objs[len(srcs):])):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [nvcc] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + lib_objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills / smem per kernel")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, ptxas_info=args.ptxas_info))
