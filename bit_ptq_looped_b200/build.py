"""Build the lq shared library (liblq.so) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "liblq.so")
# host-side sanitizer build (AddressSanitizer + UndefinedBehaviorSanitizer on
# the C++ of the library; the device code is unchanged), loaded instead of
# liblq.so when LQ_LIB_PATH points at it
LIB_SAN = os.path.join(HERE, "liblq_san.so")
# bounds-check build: kernels test their store indices and record violations
LIB_BOUNDS = os.path.join(HERE, "liblq_bounds.so")
SAN_FLAGS = ["-Xcompiler", "-fsanitize=address,-fsanitize=undefined,-fno-omit-frame-pointer,-g",
             "-lasan", "-lubsan"]
SOURCES = ["lq_api.cu", "lq_quant.cu", "lq_gemm.cu", "lq_gemv.cu", "lq_cta.cu", "lq_noalloc.cu"]
HEADERS = ["lq_common.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-Wall",
    "-shared", "-cudart", "static",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "lq.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags=None, lib: str = LIB) -> str:
    if not force and not _stale(lib):
        return lib
    cmd = [_nvcc(), *NVCC_FLAGS, *(extra_flags or []), "-I", INCLUDE, "-o", lib + ".tmp",
           *[os.path.join(CSRC, f) for f in SOURCES]]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


def build_sanitized(force: bool = False) -> str:
    """liblq_san.so: the same sources with the host code under ASan + UBSan."""
    return build(force=force, extra_flags=SAN_FLAGS, lib=LIB_SAN)


def build_bounds_checked(force: bool = False) -> str:
    """liblq_bounds.so: the kernels test their store indices (-DLQ_BOUNDS_CHECK)."""
    return build(force=force, extra_flags=["-DLQ_BOUNDS_CHECK"], lib=LIB_BOUNDS)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
    print(LIB)
