"""Build libdms.so in-tree for sm_100a with nvcc (no JIT cache, no torch extension)."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdms.so")
# The same sources with device-side bounds checks on every index the kernels
# derive (DMS_DEBUG): a bad index latches DMS_ERR_INVALID instead of faulting.
DEBUG_LIB = os.path.join(PKG, "libdms_debug.so")
SOURCES = ["dms_api.cu", "dms_append.cu", "dms_attention.cu", "dms_noalloc.cu"]
HEADERS = [os.path.join(CSRC, "dms_internal.cuh"), os.path.join(INCLUDE, "dms.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(cuda, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + HEADERS
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False, debug: bool = False) -> str:
    """Compile libdms.so (or, with debug, libdms_debug.so with DMS_DEBUG defined)."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not needs_build(lib):
        return lib
    cmd = [_nvcc()] + NVCC_FLAGS + ["-I", INCLUDE, "-o", lib]
    if debug:
        cmd += ["-DDMS_DEBUG"]
    if ptxas_info:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose=True, ptxas_info="-v" in sys.argv))
    print(build(force=True, verbose=True, debug=True))
