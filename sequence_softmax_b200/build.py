"""Build libra.so (the C-ABI library of include/ra.h) in-tree with nvcc for sm_100a.

    python -m sequence_softmax_b200.build            # build if sources are newer
    python -m sequence_softmax_b200.build --force    # always rebuild
    python -m sequence_softmax_b200.build --ptxas-info
    python -m sequence_softmax_b200.build --checked  # libra_checked.so: kernels test every
                                                     # global row index (RA_DEBUG_BOUNDS)

The library is one translation unit (csrc/ra.cu) and links the CUDA runtime statically,
so it loads next to PyTorch's own runtime and needs nothing but the NVIDIA driver.
"""

from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libra.so")
LIB_CHECKED = os.path.join(PKG, "libra_checked.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put the CUDA toolkit on PATH")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  [os.path.join(ROOT, "include", "ra.h")])


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, ptxas_info: bool = False, extra=None, checked: bool = False) -> str:
    """Build libra.so (or, with checked, libra_checked.so: the same library compiled with
    RA_DEBUG_BOUNDS, whose kernels record RA_ERR_DEVICE_BOUNDS instead of touching memory
    outside the buffers they were given). Returns the library path."""
    lib = LIB_CHECKED if checked else LIB
    if not force and not stale(lib):
        return lib
    cmd = [nvcc_path(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-I", os.path.join(ROOT, "include"), os.path.join(CSRC, "ra.cu"), "-o", lib + ".tmp"]
    if checked:
        cmd[1:1] = ["-DRA_DEBUG_BOUNDS"]
    if ptxas_info:
        cmd[1:1] = ["-Xptxas", "-v"]
    if extra:
        cmd[1:1] = list(extra)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    if ptxas_info:
        sys.stderr.write(r.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    ap.add_argument("--checked", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, ptxas_info=a.ptxas_info, checked=a.checked))


if __name__ == "__main__":
    main()
