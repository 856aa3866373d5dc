"""In-tree build of the package's shared libraries with nvcc (sm_100a).

- ``lib/libmoeq.so``        the layer library (C ABI, include/moeq.h)
- ``lib/libmoeq_synth.so``  the seeded synthetic-input generator

Both are plain ``nvcc -shared`` builds with the CUDA runtime linked
statically; the driver API (tensor maps) is reached at run time through
``cudaGetDriverEntryPoint``, so loading either library needs no GPU.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIBDIR = os.path.join(PKG, "lib")
CSRC = os.path.join(PKG, "csrc")
SYNTH = os.path.join(PKG, "synth")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
          "--expt-relaxed-constexpr", "-shared", "-cudart", "static"]


def _stale(target: str, sources: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def _nvcc(target: str, srcs: list[str], deps: list[str], extra: list[str], force: bool,
          verbose: bool) -> str:
    os.makedirs(LIBDIR, exist_ok=True)
    if not force and not _stale(target, srcs + deps):
        return target
    cmd = ["nvcc", *ARCH, *COMMON, *extra, *srcs, "-o", target + ".tmp"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(target + ".tmp", target)
    return target


def build_moeq(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False) -> str:
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    deps = sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(INCLUDE, "moeq.h")]
    extra = ["-I", INCLUDE, "-I", CSRC]
    if ptxas_verbose:
        extra += ["-Xptxas", "-v"]
    return _nvcc(os.path.join(LIBDIR, "libmoeq.so"), srcs, deps, extra, force, verbose)


def build_synth(force: bool = False, verbose: bool = False) -> str:
    srcs = [os.path.join(SYNTH, "synth.cu")]
    deps = [os.path.join(SYNTH, "synth_core.h")]
    # no fused multiply-add contraction and IEEE division: host and device
    # must round every step the same way
    extra = ["-fmad=false", "-prec-div=true", "-ftz=false", "-Xcompiler",
             "-fopenmp,-ffp-contract=off", "-lgomp"]
    return _nvcc(os.path.join(LIBDIR, "libmoeq_synth.so"), srcs, deps, extra, force, verbose)


def build_all(force: bool = False, verbose: bool = False) -> None:
    build_synth(force, verbose)
    build_moeq(force, verbose)


if __name__ == "__main__":
    build_all(force="--force" in sys.argv, verbose=True)
