"""The boundary is a C ABI: include/ra.h compiles as C99, and a C program linked against
libra.so calls it (status strings, the ABI version, argument validation that returns before
any device work), on a host without a GPU."""

import os
import shutil
import subprocess

import pytest

from sequence_softmax_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "ra.h"

int main(void) {
  if (ra_abi_version() != RA_ABI_VERSION) return 1;
  if (strncmp(ra_status_string(RA_ERR_INVALID_ARG), "RA_ERR_INVALID_ARG", 18) != 0) return 2;
  /* invalid arguments are rejected before any device work */
  if (ra_ring_forward(0, 0, 0, RA_BF16, 1, 1, 256, 128, 0.0f, 2, 1, RA_LAYOUT_ZIGZAG, 0, 0, 0) !=
      RA_ERR_INVALID_ARG) return 3;
  if (ra_merge(0, 0, 0, 16, 128, 0, RA_BF16, 0, 0) != RA_ERR_INVALID_ARG) return 4;
  if (ra_ring_backward_workspace_bytes(RA_BF16, 1, 2, 256, 128) != 2 * 256 * 4) return 5;
  if (ra_ring_backward_noalloc(0, 0, 0, 0, 0, 0, RA_BF16, 64, 64, 1 << 20, 128, 0.1f, 4, 1, RA_LAYOUT_CONTIGUOUS,
                               0, 0, 0, 0) != RA_ERR_UNSUPPORTED) return 6;
  if (ra_key_norm_max(0, RA_F32, 1, 2, 128, 128, 0, 0) != RA_ERR_UNSUPPORTED) return 7;
  if (ra_partial_fold(0, 0, 0, RA_BF16, 1, 1, -1, 128, 128, 0.1f, 0, 0, 1, 0, 1, 0, 0, 0, 0) !=
      RA_ERR_INVALID_ARG) return 8;
  printf("ok\n");
  return 0;
}
"""


def test_header_compiles_as_c_and_links():
    cc = shutil.which("gcc") or shutil.which("cc")
    cuda_inc = "/usr/local/cuda/include"
    if cc is None or not os.path.isdir(cuda_inc):
        pytest.skip("no C compiler or CUDA headers")
    build.build()
    lib_dir = os.path.dirname(binding.library_path)
    work = os.path.join(ROOT, ".pytest_cache", "c_header")
    os.makedirs(work, exist_ok=True)
    src = os.path.join(work, "use_ra.c")
    exe = os.path.join(work, "use_ra")
    with open(src, "w") as f:
        f.write(C_PROGRAM)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, src,
                        "-L", lib_dir, "-l:libra.so", "-Wl,-rpath," + lib_dir, "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
