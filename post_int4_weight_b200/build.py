"""Build libawq_b200.so (the C-ABI library of include/awq.h) for sm_100a.

    python -m post_int4_weight_b200.build [--verbose-ptxas]

Each csrc/*.cu is compiled with nvcc for sm_100a only and linked into one
shared library in the package directory, next to this file.  The FP32 rate
probe (probe/fp32_rate.cu, not part of the library or its C ABI) is built
into its own small libawq_probe.so for bench.py.  No fast-math:
the kernels rely on IEEE round-to-nearest-even fp32 division, square root and
conversions where the method's integer decisions are taken.
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libawq_b200.so")
PROBE_SRC = os.path.join(PKG, "probe", "fp32_rate.cu")
PROBE_LIB = os.path.join(PKG, "libawq_probe.so")
BUILD_DIR = os.path.join(PKG, "_build")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
         "-I" + INCLUDE, "-I" + CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (_sources() + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(CSRC, "*.h"))
            + [os.path.join(INCLUDE, "awq.h"), os.path.abspath(__file__)])


def up_to_date() -> bool:
    if not os.path.exists(LIB) or not os.path.exists(PROBE_LIB):
        return False
    t = os.path.getmtime(LIB)
    return (all(os.path.getmtime(p) <= t for p in _deps())
            and os.path.getmtime(PROBE_SRC) <= os.path.getmtime(PROBE_LIB))


def build(force: bool = False, verbose_ptxas: bool = False, jobs: int = 8) -> str:
    if not force and not verbose_ptxas and up_to_date():
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    procs = []
    objs = []
    for src in _sources():
        obj = os.path.join(BUILD_DIR, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                            stderr=subprocess.STDOUT, text=True)))
        if len(procs) >= jobs:
            _drain(procs, verbose_ptxas)
    _drain(procs, verbose_ptxas)
    tmp = LIB + ".tmp"
    subprocess.run([NVCC, *ARCH, "-shared", "-o", tmp, *objs], check=True)
    os.replace(tmp, LIB)
    tmp = PROBE_LIB + ".tmp"
    subprocess.run([NVCC, *ARCH, "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
                    PROBE_SRC, "-o", tmp], check=True)
    os.replace(tmp, PROBE_LIB)
    return LIB


def _drain(procs, echo):
    for cmd, p in procs:
        out, _ = p.communicate()
        if p.returncode != 0:
            sys.stderr.write(out)
            raise RuntimeError("nvcc failed: " + " ".join(cmd))
        if echo and out:
            sys.stdout.write(out)
    procs.clear()


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas))
