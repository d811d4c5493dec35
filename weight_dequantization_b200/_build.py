"""In-tree build of the native libraries of this package.

``liblt_decode.so``  CUDA kernels + C ABI, compiled for sm_100a only.
``synth/liblt_synth.so``  host input generator (plain C, pthreads).
"""
from __future__ import annotations

import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
DECODE_LIB = os.path.join(PKG, "liblt_decode.so")
SYNTH_LIB = os.path.join(PKG, "synth", "liblt_synth.so")

# CUDA sources, plus the host-only container header code (lt_hct.cpp, built
# by nvcc's host compiler into the same library)
CUDA_SOURCES = ["lt_abi.cu", "lt_dequant.cu", "lt_dict.cu", "lt_zrle.cu", "lt_lz4.cu", "lt_xxh3.cu", "lt_gemm.cu",
                "lt_hct.cpp"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def _newer(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(d) <= t for d in deps)


def build_decode(force: bool = False, verbose_ptxas: bool = False) -> str:
    """Compile the CUDA sources into ``liblt_decode.so`` (sm_100a)."""
    srcs = [os.path.join(CSRC, s) for s in CUDA_SOURCES]
    hdrs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hdrs.append(os.path.join(ROOT, "include", "lt_decode.h"))
    if not force and _newer(DECODE_LIB, srcs + hdrs):
        return DECODE_LIB
    nvcc = _nvcc()
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for s in srcs:
        o = os.path.join(objdir, os.path.basename(s) + ".o")
        cmd = [nvcc, *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-c", s, "-o", o]
        if verbose_ptxas:
            cmd += ["-Xptxas", "-v"]
        subprocess.run(cmd, check=True)
        objs.append(o)
    tmp = DECODE_LIB + ".tmp"
    subprocess.run([nvcc, *NVCC_FLAGS, "-shared", *objs, "-o", tmp], check=True)
    os.replace(tmp, DECODE_LIB)
    return DECODE_LIB


def build_synth(force: bool = False) -> str:
    """Compile the host input generator into ``synth/liblt_synth.so``."""
    src = os.path.join(PKG, "synth", "lt_synth.c")
    if not force and _newer(SYNTH_LIB, [src]):
        return SYNTH_LIB
    tmp = SYNTH_LIB + ".tmp"
    subprocess.run(["gcc", "-O2", "-std=gnu11", "-fPIC", "-shared", "-fvisibility=hidden",
                    src, "-o", tmp, "-lm", "-lpthread"], check=True)
    os.replace(tmp, SYNTH_LIB)
    return SYNTH_LIB


def build_all(force: bool = False) -> None:
    build_synth(force)
    build_decode(force)
