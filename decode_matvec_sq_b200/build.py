"""Builds the in-tree CUDA libraries with nvcc for sm_100a.

    python -m decode_matvec_sq_b200.build          # libsq.so + libsqsynth.so

* ``decode_matvec_sq_b200/libsq.so``: the product library (include/sq.h).
* ``synth/libsqsynth.so``: the device generator of the synthetic inputs.

Both link the CUDA runtime dynamically so that they share one runtime (and one
notion of the current device) with PyTorch in the same process.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIBSQ = os.path.join(PKG, "libsq.so")
LIBSYNTH = os.path.join(ROOT, "synth", "libsqsynth.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
                 "-I" + os.path.join(ROOT, "include")]

# (source, extra flags).  The decomposition and the activation split must
# reproduce an exact operation sequence: no multiply-add contraction there.
SOURCES = [
    ("sq_api.cu", []),
    ("sq_pack.cu", ["-fmad=false"]),
    ("sq_act.cu", ["-fmad=false"]),
    ("sq_linear.cu", []),
    ("sq_linear_tc.cu", []),
    ("sq_noalloc.cu", []),
    ("sq_prefill.cu", []),
    ("sq_nvfp4.cu", ["-fmad=false"]),
    ("sq_probe.cu", []),
]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libsq")


def _newer(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)


def build_libsq(force: bool = False, verbose: bool = False, ptxas_v: bool = False) -> str:
    nvcc = _nvcc()
    os.makedirs(BUILD, exist_ok=True)
    headers = [os.path.join(CSRC, h) for h in os.listdir(CSRC) if h.endswith((".h", ".cuh"))]
    headers.append(os.path.join(ROOT, "include", "sq.h"))
    objs = []
    for src, extra in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _newer(o, [s] + headers + [__file__]):
            flags = COMMON + extra + (["-Xptxas", "-v"] if ptxas_v else [])
            _run([nvcc, *flags, "-c", s, "-o", o], verbose)
    if force or _newer(LIBSQ, objs):
        tmp = LIBSQ + ".tmp.%d" % os.getpid()
        _run([nvcc, *ARCH, "-shared", "-cudart", "shared", "-o", tmp, *objs], verbose)
        os.replace(tmp, LIBSQ)
    return LIBSQ


def build_synth(force: bool = False, verbose: bool = False) -> str:
    nvcc = _nvcc()
    src = os.path.join(ROOT, "synth", "synth_dev.cu")
    if force or _newer(LIBSYNTH, [src, __file__]):
        tmp = LIBSYNTH + ".tmp.%d" % os.getpid()
        _run([nvcc, *COMMON, "-fmad=false", "-shared", "-cudart", "shared", "-o", tmp, src], verbose)
        os.replace(tmp, LIBSYNTH)
    return LIBSYNTH


def build_all(force: bool = False, verbose: bool = False) -> None:
    build_libsq(force=force, verbose=verbose)
    build_synth(force=force, verbose=verbose)


if __name__ == "__main__":
    build_all(force="--force" in sys.argv, verbose=True)
    if "--ptxas" in sys.argv:
        build_libsq(force=True, verbose=True, ptxas_v=True)
