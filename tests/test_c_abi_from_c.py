"""The C ABI is usable from plain C: a C99 program that includes only
include/moe_mxfp8.h, links the library and calls its host-side entry points
(sizes, status strings, argument checks -- nothing that needs a device)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "moe_mxfp8.h"

int main(void) {
  int bad = 0;
  if (moe_padded_rows(512, 2, 4) != 1536) bad |= 1;
  if (moe_mx_scale_bytes(1, 128, 128) != 512) bad |= 2;
  if (moe_mx_scale_bytes(1, 128, 100) != -1) bad |= 4;
  if (moe_workspace_size(MOE_OP_FWD, 512, 2, 4, 256, 512) <= 0) bad |= 8;
  if (strlen(moe_status_string(MOE_ERR_TIMEOUT)) == 0) bad |= 16;
  /* rejected on the host before any device work */
  if (moe_combine(NULL, 4, 2, 64, NULL, NULL) != MOE_ERR_INVALID) bad |= 32;
  if (moe_router_topk(NULL, MOE_DTYPE_F32, 4, 8, 2, NULL, NULL, NULL) != MOE_ERR_INVALID) bad |= 64;
  printf("%d\n", bad);
  return bad;
}
"""


def test_c_program_links_and_calls_the_library(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    from mxfp8_grouped_gemm_x32_b200 import build_lib
    so = build_lib.build()
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(so)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), so, f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, (out.stdout, out.stderr)
    assert out.stdout.strip() == "0"
