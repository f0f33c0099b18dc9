"""Build librope3d.so in-tree with nvcc for sm_100a (B200).

    python -m rotary_position_encoding_b200.build [--force] [--checked]

--checked also builds librope3d_checked.so: the same library compiled with
-DROPE3D_DEVICE_CHECKS, whose step kernels test every cache, table and destination row
they derive and report a row outside its extent as ROPE3D_EINDEX instead of touching it.

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
CHECKED_LIBRARY = os.path.join(PKG, "librope3d_checked.so")
CHECKED_FLAGS = ("-DROPE3D_DEVICE_CHECKS",)
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


def _command(library: str, extra_flags):
    tmp = library + ".tmp%d" % os.getpid()
    return tmp, [nvcc(), *NVCC_FLAGS, *extra_flags, "-I", INCLUDE, "-I", CSRC, *SOURCES, "-o",
                 tmp]


def build(force: bool = False, library: str = LIBRARY, extra_flags=(), verbose: bool = False) -> str:
    if not force and not stale(library):
        return library
    tmp, cmd = _command(library, extra_flags)
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, library)
    return library


def build_all(force: bool = False, verbose: bool = False):
    """librope3d.so and librope3d_checked.so, compiled side by side."""
    jobs = [(lib, flags) for lib, flags in ((LIBRARY, ()), (CHECKED_LIBRARY, CHECKED_FLAGS))
            if force or stale(lib)]
    procs = []
    for lib, flags in jobs:
        tmp, cmd = _command(lib, flags)
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((lib, tmp, subprocess.Popen(cmd)))
    failed = [lib for lib, tmp, proc in procs if proc.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, "nvcc: " + ", ".join(failed))
    for lib, tmp, _ in procs:
        os.replace(tmp, lib)
    return LIBRARY, CHECKED_LIBRARY


if __name__ == "__main__":
    if "--checked" in sys.argv:
        print(*build_all(force="--force" in sys.argv, verbose=True))
    else:
        print(build(force="--force" in sys.argv, verbose=True))
