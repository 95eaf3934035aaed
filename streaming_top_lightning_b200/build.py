"""Build the CUDA library libstreamindex.so in-tree with nvcc for sm_100a.

    python -m streaming_top_lightning_b200.build [--force] [--debug]

The library is a plain shared object with a C ABI (include/streamindex.h);
the CUDA runtime is linked statically so the library does not depend on the
runtime version PyTorch ships.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libstreamindex.so")
# profiling build: the same sources with per-role cycle counters (SI_ROLE_CLOCKS)
LIB_ROLES = os.path.join(PKG, "libstreamindex_roles.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps += glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, debug: bool = False, verbose: bool = False,
          roles: bool = False) -> str:
    """Compile every .cu under csrc/ into libstreamindex.so (skipped when up to
    date); ``roles`` builds the profiling variant libstreamindex_roles.so."""
    lib = LIB_ROLES if roles else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH, "-lineinfo", "-O3", "-std=c++17", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC", "-shared", "--cudart", "static", "-I", INCLUDE, "-I", CSRC,
           "-o", tmp, *sources()]
    if debug:
        cmd.insert(1, "-DSI_DEBUG")
    if roles:
        cmd.insert(1, "-DSI_ROLE_CLOCKS")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, debug="--debug" in sys.argv,
                verbose="-v" in sys.argv, roles="--roles" in sys.argv))
