"""Builds libvsa.so (the product library) and the test-only tcgen05 check
library in-tree with nvcc for sm_100a. Run as a script or call build()."""

from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3",
                     "-I" + INCLUDE, "-I" + CSRC]

LIBVSA_SOURCES = ["vsa_layout.cpp", "vsa_select.cu", "vsa_select_tc.cu", "vsa_attn.cu", "vsa_extra.cu", "vsa_bwd.cu"]
LIBVSA = os.path.join(PKG, "libvsa.so")
CHECK_SOURCE = os.path.join(ROOT, "tests", "native", "mma_check.cu")
CHECK_LIB = os.path.join(ROOT, "tests", "native", "libmma_check.so")


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("command failed: %s\n%s\n%s" % (" ".join(cmd), r.stdout, r.stderr))
    return r


def _newer(target, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _headers():
    hs = [os.path.join(INCLUDE, "vsa.h")]
    hs += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    return hs


def build(verbose: bool = False, force: bool = False) -> None:
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    headers = _headers()
    objs, jobs = [], []
    for src in LIBVSA_SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        objs.append(o)
        if force or _newer(o, [s] + headers):
            jobs.append([nvcc] + NVCC_FLAGS + ["-c", s, "-o", o])
    with ThreadPoolExecutor(len(jobs) or 1) as ex:
        for r in ex.map(_run, jobs):
            if verbose and r.stderr:
                print(r.stderr, file=sys.stderr)
    if force or jobs or _newer(LIBVSA, objs):
        _run([nvcc] + ARCH + ["-shared", "-o", LIBVSA] + objs)
    if force or _newer(CHECK_LIB, [CHECK_SOURCE] + headers):
        _run([nvcc] + NVCC_FLAGS + ["-shared", CHECK_SOURCE, "-o", CHECK_LIB])


if __name__ == "__main__":
    build(verbose=True, force="--force" in sys.argv)
    print(LIBVSA)
