"""Build libfvattn.so in-tree with nvcc for sm_100a (B200).

    python -m block_sparse_top_fvattn_b200.build [--verbose-ptxas] [--debug]

--debug builds libfvattn_debug.so instead: the same sources with -DFVATTN_DEBUG, whose kernels
check every CSR list before reading it (offsets within the column array, key blocks in range,
lists ascending) and report a failed check as FVATTN_ERR_INVALID in the device status word.

The CUDA runtime is linked statically, so the library loads (and its host-only entry points
work) on machines without a GPU or driver; device code is sm_100a only.
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
LIB = os.path.join(PKG, "libfvattn.so")
DEBUG_LIB = os.path.join(PKG, "libfvattn_debug.so")

SOURCES = ["api.cu", "route.cu", "attn_f32.cu", "attn_tc.cu", "route_static.cu", "balance.cu", "score_tc.cu"]
HEADERS = ["common.cuh", "route.cuh", "route_dev.cuh", "tc_ptx.cuh", "tmap.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False) -> str:
    bdir = os.path.join(BUILD, "debug") if debug else BUILD
    lib = DEBUG_LIB if debug else LIB
    os.makedirs(bdir, exist_ok=True)
    headers = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "fvattn.h")]
    objs = []
    procs = []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(bdir, src.replace(".cu", ".o"))
        objs.append(o)
        if force or verbose_ptxas or _stale(o, [s] + headers):
            cmd = [nvcc(), *NVCC_FLAGS, *(["-DFVATTN_DEBUG"] if debug else []), "-I", INCLUDE, "-I", CSRC, "-c", s,
                   "-o", o]
            if verbose_ptxas:
                cmd += ["-Xptxas", "-v"]
            procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        text = out.decode(errors="replace")
        if p.returncode != 0:
            failed.append(src)
            sys.stderr.write(text)
        elif verbose_ptxas:
            sys.stdout.write(text)
    if failed:
        raise RuntimeError(f"nvcc failed for {failed}")
    if force or _stale(lib, objs):
        cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
               "-Xcompiler", "-fPIC", *objs, "-o", lib]
        subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--debug", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas, debug=a.debug))
