"""Build libq4.so (the C-ABI library) in-tree with nvcc for sm_100a.

The CUDA runtime is linked statically and the tensor-map encoder is looked up
through the runtime's driver entry-point query, so the library loads on
machines without a GPU driver (calls then fail with Q4_ERR_CUDA).
"""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
CSRC = PKG / "csrc"
INCLUDE = PKG.parent / "include"
LIB = PKG / "libq4.so"
SOURCES = ["q4_api.cu", "q4_quant.cu", "q4_gemm.cu", "q4_noalloc.cu"]
HEADERS = ["q4_internal.h", "q4_codec.cuh", "q4_ptx.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    # no contraction of a plain multiply and add into one fused operation:
    # the codecs' decisions depend on every intermediate rounding (intended
    # fused operations are written as explicit fma).  This does not stop
    # ptxas from fusing a paired (f32x2) multiply into a paired add, so the
    # kernels keep the product that feeds such an add scalar where it matters
    "-fmad=false",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-cudart", "static",
]


def nvcc() -> str:
    cand = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    p = Path(cand) / "bin" / "nvcc"
    return str(p) if p.exists() else "nvcc"


def _stale() -> bool:
    if not LIB.exists():
        return True
    t = LIB.stat().st_mtime
    deps = [CSRC / s for s in SOURCES + HEADERS] + [INCLUDE / "q4.h", Path(__file__)]
    return any(d.stat().st_mtime > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=None) -> Path:
    """Compile every source to an object and link the shared library."""
    if not force and not _stale():
        return LIB
    objdir = PKG / "_build"
    objdir.mkdir(exist_ok=True)
    objs, procs = [], []
    # the sources compile independently: one nvcc process each, in parallel
    for src in SOURCES:
        obj = objdir / (Path(src).stem + ".o")
        cmd = [nvcc(), *NVCC_FLAGS, *(extra or []), "-I", str(INCLUDE), "-c",
               str(CSRC / src), "-o", str(obj)]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((cmd, subprocess.Popen(cmd)))
        objs.append(str(obj))
    for cmd, proc in procs:
        if proc.wait() != 0:
            raise subprocess.CalledProcessError(proc.returncode, cmd)
    tmp = LIB.with_suffix(f".{os.getpid()}.tmp")
    cmd = [nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-cudart", "static",
           "-Xcompiler", "-fPIC", *objs, "-o", str(tmp)]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas" in sys.argv else None)
    print(LIB)
