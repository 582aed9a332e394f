"""include/pqk.h is a plain C header: a C99 translation unit that includes it
compiles with -Wall -Wextra -pedantic -Werror, links against libpqk.so and
runs the host-side contract (status strings, version, workspace sizes,
argument errors returned before anything is enqueued) without a GPU and
without the Python binding."""

import os
import shutil
import subprocess

import pytest

from packed_attention_qk_b200 import build as pqk_build
from packed_attention_qk_b200 import pqk

C_SRC = r'''
#include <math.h>
#include <stdio.h>
#include <string.h>
#include "pqk.h"

int main(void) {
  void* a = (void*)0x10000;                  /* aligned fake device address, never dereferenced */
  int fails = 0;
  if (strcmp(pqk_status_string(PQK_OK), "ok") != 0) ++fails;
  if (pqk_version() == NULL || strlen(pqk_version()) < 5) ++fails;
  if (pqk_varlen_attn_workspace_size(0) != 0) ++fails;
  if (pqk_varlen_attn_workspace_size(4096) < pqk_varlen_attn_workspace_size(1)) ++fails;
  /* argument errors are host-side and need no GPU */
  if (pqk_qk_norm_rope(a, a, a, a, 1024, 1024, 1024, 1024, a, a, a, 16, 8, 96, 1e-6f, 1e4f, 0, NULL) !=
      PQK_ERR_UNSUPPORTED)
    ++fails;
  if (pqk_varlen_attn_fwd(a, a, a, a, NULL, 1024, 1024, 1024, 1024, a, 0, 512, 8, 128, 0.1f, a, 4096, NULL) !=
      PQK_ERR_INVALID_ARG)
    ++fails;
  if (pqk_varlen_attn_fwd_skip(a, a, a, a, NULL, 1024, 1024, 1024, 1024, a, 2, 512, 8, 128, 0.1f, -1.0f, NULL, a,
                               4096, NULL) != PQK_ERR_INVALID_ARG)
    ++fails;
  if (pqk_varlen_attn_fwd_fp8qk(a, a, a, a, a, NULL, 512, 512, a, 2, 512, 8, 64, 0.1f, INFINITY, NULL, a, 4096,
                                NULL) != PQK_ERR_UNSUPPORTED)
    ++fails;
  if (pqk_quantize_qk_e4m3(a, a, 1024, 1024, 16, 8, 128, a, a, NULL, NULL) != PQK_ERR_INVALID_ARG) ++fails;
  if (pqk_modulate_swiglu(a, NULL, NULL, a, a, a, NULL, a, 1, 8, 250, 0, 1e-6f, NULL, NULL, 0, NULL, 0, NULL) !=
      PQK_ERR_INVALID_ARG)
    ++fails;
  if (pqk_varlen_attn_fwd_noalloc(a, a, a, a, NULL, 1024, 1024, 1024, 1024, a, 5000, 512, 8, 128, 0.1f, NULL) !=
      PQK_ERR_WORKSPACE)
    ++fails;
  if (pqk_linear_gated_residual(a, 256, a, a, 512, NULL, a, 2, a, 512, 300, 256, 512, NULL) != PQK_ERR_INVALID_ARG)
    ++fails;
  if (pqk_linear_swiglu(a, 256, a, (void*)0x10004, 512, 300, 256, 512, NULL) != PQK_ERR_MISALIGNED) ++fails;
  printf("%d\n", fails);
  return fails != 0;
}
'''


def test_header_compiles_as_c99_and_the_host_contract_holds(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    pqk_build.build()
    src = tmp_path / "abi.c"
    src.write_text(C_SRC)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(pqk.LIB_PATH)
    subprocess.check_call([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", pqk_build.INCLUDE,
                           str(src), "-o", str(exe), "-L", libdir, "-l:libpqk.so", f"-Wl,-rpath,{libdir}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "0"
