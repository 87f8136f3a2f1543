"""Build the CUDA libraries in-tree for sm_100a with nvcc.

    python -m gated_deltanet_cpr_delta_b200.build [--force] [--verbose]

libgdn_cpr.so is the layer (the C ABI of include/gdn_cpr.h).  libgdn_probe.so
is a measurement helper for the benchmark (the FP32 fma rate of the device).
`--verbose` adds ``-Xptxas -v`` (registers, spills, shared memory per kernel).
"""
from __future__ import annotations

import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libgdn_cpr.so")
PROBE_LIB = os.path.join(PKG, "libgdn_probe.so")
PROBE_SOURCES = ["probe_fp32.cu"]
SOURCES = ["gdn_cpr.cu", "identity.cu"]
DEPS = ["gdn_cpr.cu", "identity.cu", "kernels.cuh", "schedule.cuh", "tma.cuh", "k_tables.cuh", "k_ptok.cuh",
        "k_tc.cuh", "k_prep.cuh", "k_pchunk.cuh", "k_decode.cuh", "k_bwd.cuh", "k_bgrad.cuh"]
HEADERS = [os.path.join(ROOT, "include", "gdn_cpr.h")]


def sources_sha256() -> str:
    """SHA-256 over the library's sources (file name, NUL, contents, in DEPS
    order, then the public header): the deployment identity names it."""
    h = hashlib.sha256()
    for path in [os.path.join(CSRC, s) for s in DEPS] + HEADERS:
        h.update(os.path.basename(path).encode() + b"\0")
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(verbose: bool = False):
    f = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-Xcompiler", "-fPIC", "-shared",
         # the schedule's arithmetic is written with explicit _rn intrinsics;
         # these keep any other fp expression exact too
         "-fmad=false", "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
         "-I", os.path.join(ROOT, "include"), "-I", CSRC,
         f'-DGDN_SOURCES_SHA256="{sources_sha256()}"']
    if verbose:
        f += ["-Xptxas", "-v"]
    return f


def up_to_date(lib: str, deps) -> bool:
    if not os.path.exists(lib):
        return False
    m = os.path.getmtime(lib)
    srcs = [os.path.join(CSRC, s) for s in deps] + HEADERS + [os.path.abspath(__file__)]
    return all(os.path.getmtime(s) <= m for s in srcs)


def _nvcc(lib: str, sources, verbose: bool):
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), *flags(verbose), *[os.path.join(CSRC, s) for s in sources], "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or verbose or not up_to_date(LIB, DEPS):
        _nvcc(LIB, SOURCES, verbose)
    if force or verbose or not up_to_date(PROBE_LIB, PROBE_SOURCES):
        _nvcc(PROBE_LIB, PROBE_SOURCES, verbose)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
