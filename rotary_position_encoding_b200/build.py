"""Build librope3d.so in-tree with nvcc for sm_100a (B200).

    python -m rotary_position_encoding_b200.build [--force]

The CUDA runtime is linked statically, so the library does not depend on which
libcudart another library in the process (for example PyTorch) loaded; device memory,
streams and the current device are shared through the driver.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "librope3d.so")
SOURCES = [os.path.join(CSRC, "rope3d.cu")]
DEPENDS = SOURCES + [os.path.join(CSRC, f) for f in ("rope3d_kernels.cuh", "rope3d_tma.cuh",
                                                    "rope3d_gemm.cuh")] + \
    [os.path.join(INCLUDE, f) for f in ("rope3d.h", "rope3d_testing.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build librope3d.so")
    return path


def stale(library: str = LIBRARY) -> bool:
    if not os.path.exists(library):
        return True
    built = os.path.getmtime(library)
    return any(os.path.getmtime(d) > built for d in DEPENDS)


def build(force: bool = False, library: str = LIBRARY, extra_flags=(), verbose: bool = False) -> str:
    if not force and not stale(library):
        return library
    tmp = library + ".tmp%d" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, *extra_flags, "-I", INCLUDE, "-I", CSRC, *SOURCES, "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, library)
    return library


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
