"""Build libb200attn.so in-tree with nvcc for sm_100a.

``python -m long_context_bidirectional_b200.build`` (or ``build()``) compiles
``csrc/b200attn.cu`` into ``long_context_bidirectional_b200/lib/``.  The CUDA
runtime is linked statically so the library loads on a host without a GPU
(entry points then return B2A_ERR_CUDA).  Rebuilds only when a source or
the header is newer than the library, unless ``force``.
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
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libb200attn.so")
# The debug build (-DB2A_DEBUG): every TMA box and TMEM access bounds-checked
# on the device before issue; selected in the binding by ATTN_DEBUG=1.
DEBUG_LIB = os.path.join(LIBDIR, "libb200attn_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libb200attn.so")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(CSRC, "*.h"))
                  + [os.path.join(INCLUDE, "b200attn.h")])


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug: bool = False) -> str:
    """Compile the release library, or with ``debug`` the bounds-checked one."""
    lib = DEBUG_LIB if debug else LIB
    if not force and up_to_date(lib):
        return lib
    os.makedirs(LIBDIR, exist_ok=True)
    tmp = lib + ".tmp"
    if debug:
        extra_flags = ("-DB2A_DEBUG", *extra_flags)
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-shared", "-cudart", "static", f"-I{INCLUDE}", f"-I{CSRC}",
           "-DB2A_BUILDING_LIBRARY", *extra_flags,
           os.path.join(CSRC, "b200attn.cu"), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose:
        print(res.stderr, file=sys.stderr)
    os.replace(tmp, lib)
    return lib


def build_all(force: bool = False) -> None:
    """Both libraries, compiled concurrently."""
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(2) as ex:
        for f in [ex.submit(build, force, False, (), dbg) for dbg in (False, True)]:
            f.result()


if __name__ == "__main__":
    force = "--force" in sys.argv
    if "--debug" in sys.argv:
        print(build(force=force, verbose="-v" in sys.argv, debug=True))
    else:
        print(build(force=force, verbose="-v" in sys.argv))
