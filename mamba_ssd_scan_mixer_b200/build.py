"""Build libmamba2ssd.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m mamba_ssd_scan_mixer_b200.build [--force] [--checked]

The library is plain CUDA C++ with a C ABI (include/mamba2ssd.h); it links
the CUDA runtime statically and needs no PyTorch at build time.  --checked
also builds libmamba2ssd_checked.so, the same library compiled with
-DMAMBA2_BOUNDS_CHECK: every plain global access of the tensor-core prefill and
decode kernels is checked against its buffer's extent and alignment, skipped if
it fails, and reported by mamba2_device_errors (bit 1).  Load it by setting
MAMBA2SSD_LIBRARY to its path before importing the binding.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
INCLUDE = os.path.join(ROOT, "include")
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmamba2ssd.so")
LIB_CHECKED = os.path.join(PKG, "libmamba2ssd_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Build the library (or, with checked, its bounds-checked twin); returns its path."""
    lib = LIB_CHECKED if checked else LIB
    if not force and not _stale(lib):
        return lib
    objdir = os.path.join(ROOT, "_build", "checked" if checked else "release")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    extra = ["-DMAMBA2_BOUNDS_CHECK"] if checked else []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.run([nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-o", tmp, *objs, "-lcuda"], check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    if "--checked" in sys.argv:
        print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, checked=True))
