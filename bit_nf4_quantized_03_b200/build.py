"""Builds libqlora.so in-tree with nvcc for sm_100a.

    python -m bit_nf4_quantized_03_b200.build [--force] [--verbose] [--bounds-check]

Objects go to bit_nf4_quantized_03_b200/_build/, the shared library to
bit_nf4_quantized_03_b200/libqlora.so. A rebuild happens only when a source
or header is newer than the library (or with --force).

--bounds-check builds libqlora_bounds.so (objects in _build_bounds/) with
-DQLORA_BOUNDS_CHECK: the kernels check every TMA tile start (16-byte
alignment of the innermost coordinate, range), every bulk copy and the main
global stores, and record a failure in the device error word (with the site
number) instead of making the access. The binding loads it instead of
libqlora.so when QLORA_BOUNDS_CHECK=1 is set in the environment.
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libqlora.so")
BUILD_BOUNDS = os.path.join(PKG, "_build_bounds")
LIB_BOUNDS = os.path.join(PKG, "libqlora_bounds.so")
SOURCES = ["nf4_quant.cu", "nf4_gemm.cu", "nf4_wgemm.cu", "elementwise.cu", "qlora_abi.cu", "nf4_merge.cu", "dropout.cu", "optim.cu", "qlora_noalloc.cu"]
HEADERS = ["qlora_device.cuh", "qlora_kernels.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-rdc=true", "-Xcompiler", "-fPIC",
              "-Xptxas", "-v", "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _newest_input() -> float:
    paths = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    paths.append(os.path.join(ROOT, "include", "qlora.h"))
    paths.append(os.path.abspath(__file__))
    return max(os.path.getmtime(p) for p in paths)


def build(force: bool = False, verbose: bool = False, bounds_check: bool = False) -> str:
    lib, bdir = (LIB_BOUNDS, BUILD_BOUNDS) if bounds_check else (LIB, BUILD)
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= _newest_input():
        return lib
    os.makedirs(bdir, exist_ok=True)
    nvcc = _nvcc()
    extra = ["-DQLORA_BOUNDS_CHECK"] if bounds_check else []
    procs = []
    for src in SOURCES:
        obj = os.path.join(bdir, src.replace(".cu", ".o"))
        cmd = [nvcc, *ARCH, *NVCC_FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
        procs.append((src, obj, cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                                      text=True)))
    objs = []
    for src, obj, cmd, pr in procs:
        out, _ = pr.communicate()
        if pr.returncode != 0:
            sys.stderr.write(out)
            raise RuntimeError(f"nvcc failed on {src}: {' '.join(cmd)}")
        if verbose:
            sys.stdout.write(out)
        with open(os.path.join(bdir, src.replace(".cu", ".ptxas.txt")), "w") as f:
            f.write(out)
        objs.append(obj)
    tmp = lib + ".tmp"
    cmd = [nvcc, *ARCH, "-shared", "-rdc=true", "-Xcompiler", "-fPIC", *objs, "-o", tmp]
    r = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout)
        raise RuntimeError("link failed: " + " ".join(cmd))
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--bounds-check", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, bounds_check=a.bounds_check))
