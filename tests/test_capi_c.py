"""The C ABI from plain C: include/nabla.h compiles as C99 and a C program links against
libnabla.so and calls it (host-side calls only: sizes, status strings and a call that
fails its argument checks before anything reaches the GPU)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "nabla.h"

int main(void) {
  nabla_shape s;
  memset(&s, 0, sizeof(s));
  s.B = 1; s.H = 2; s.T = 2; s.Hg = 16; s.W = 16; s.D = 64; s.P = 8;
  if (nabla_mask_workspace_bytes(s) <= 256) return 1;
  if (nabla_fwd_workspace_bytes(s) == 0) return 2;
  if (strcmp(nabla_status_string(NABLA_ERR_WORKSPACE), "NABLA_ERR_WORKSPACE") != 0) return 3;
  s.Hg = 12;   /* not a multiple of the patch size */
  if (nabla_reorder((const void*)0x10000, NABLA_BF16, (void*)0x20000000, NABLA_BF16, NULL, s, 0,
                    NULL) != NABLA_ERR_INVALID_ARG)
    return 4;
  printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_program_links_and_calls_the_library(tmp_path):
    from adaptive_block_sparse_b200 import build as b
    b.build()
    libdir = os.path.join(ROOT, "adaptive_block_sparse_b200")
    src = tmp_path / "main.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "main"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lnabla", f"-Wl,-rpath,{libdir}"],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.strip() == "ok"
