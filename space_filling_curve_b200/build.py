"""Compile libtess.so in-tree with nvcc for sm_100a (B200)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libtess.so")
SOURCES = ["capi.cu", "hilbert_sort.cu", "neighbors.cu", "step.cu", "static_scratch.cu", "step_graph.cu"]
HEADERS = ["common.cuh", "scan.cuh", "hilbert_table.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-O2",
    "-I", INCLUDE,
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


# Build variants: the product library, and two diagnostic builds with the
# same entry points -- "check" (-DTESS_CHECK: kernels test the indices they
# scatter to or gather from, record a bad one in the caller's status word and
# skip the access) and "nvtx" (-DTESS_NVTX: an NVTX range per stage).  Select
# a variant at run time with TESS_LIBRARY=<path of its .so>.
VARIANTS = {None: [], "check": ["-DTESS_CHECK"], "nvtx": ["-DTESS_NVTX"]}


def library_for(variant: str | None = None) -> str:
    return LIB if variant is None else os.path.join(HERE, "libtess_%s.so" % variant)


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "tess.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          variant: str | None = None) -> str:
    lib = library_for(variant)
    if not force and not _stale(lib):
        return lib
    objdir = os.path.join(HERE, "_build" if variant is None else "_build_%s" % variant)
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        cmd = [nvcc(), *NVCC_FLAGS, *VARIANTS[variant], *(extra or []), "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = lib + ".tmp.%d" % os.getpid()
    subprocess.check_call([nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", *objs, "-o", tmp,
                           "-lcudart"])
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    v = None
    for a in sys.argv[1:]:
        if a.startswith("--variant="):
            v = a.split("=", 1)[1]
    print(build(force="--force" in sys.argv, verbose=True,
                extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None, variant=v))
