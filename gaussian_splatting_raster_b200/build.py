"""Build libsplat.so in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libsplat.so")
LIB_CHECKED = os.path.join(PKG, "libsplat_checked.so")  # bounds-checked build (-DSPLAT_CHECKED)
SOURCES = ["capi.cu", "project.cu", "binning.cu", "raster.cu", "finalize.cu", "backward.cu",
           "attributes.cu", "noalloc.cu"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    # the decision path relies on explicit, correctly rounded fp32 operations
    "-fmad=false", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def sources() -> list[str]:
    return [os.path.join(CSRC, s) for s in SOURCES]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    deps = sources() + [os.path.join(CSRC, "common.cuh"), os.path.join(CSRC, "traverse.cuh"),
                        os.path.join(ROOT, "include", "splat.h")]
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Compile libsplat.so (or, with checked=True, the bounds-checked libsplat_checked.so)."""
    lib = LIB_CHECKED if checked else LIB
    if not force and up_to_date(lib):
        return lib
    cmd = [nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), *sources(), "-o", lib + ".tmp"]
    if checked:
        cmd.insert(1, "-DSPLAT_CHECKED")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    import sys
    print(build(force=True, verbose="-v" in sys.argv, checked="--checked" in sys.argv))
