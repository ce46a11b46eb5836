"""The boundary is a plain C ABI: a C program compiled with gcc against
include/tsa.h links libtsa.so and uses the host-side calls (no GPU needed)."""

import os
import shutil
import subprocess

import pytest

from long_context_tsa_b200 import _native as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <stdio.h>
#include <string.h>
#include "tsa.h"

int main(void) {
  tsa_desc d = {1, 32, 8, 8192, 128, TSA_BF16, 0.0f};
  size_t ws = tsa_workspace_size(&d, 64);
  if (ws < 256) return 1;
  tsa_desc bad = d;
  bad.D = 96;
  if (tsa_workspace_size(&bad, 64) != 0) return 2;
  if (strcmp(tsa_status_string(TSA_OK), tsa_status_string(TSA_ERR_INVALID_ARG)) == 0) return 3;
  /* argument errors come back before anything touches a device */
  int32_t budgets[8] = {4096, 4096, 4096, 4096, 4096, 4096, 4096, 0};
  void* fake = (void*)0x100000;
  if (tsa_select(&d, (const float*)fake, budgets, (int32_t*)fake, fake, 1 << 20, NULL) != TSA_ERR_INVALID_ARG)
    return 4;
  if (tsa_select_coverage(&d, (const float*)fake, 1.5, (int32_t*)fake, (int32_t*)fake, fake, 1 << 20, NULL) !=
      TSA_ERR_INVALID_ARG)
    return 5;
  double hist[4] = {0.9, 0.05, 0.04, 0.03};
  int32_t stable = -1;
  if (tsa_layer_stable(hist, 4, 3, 0.1, &stable) != TSA_OK || stable != 1) return 6;
  if (tsa_drift_workspace_size() < 256) return 7;
  printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_links_and_calls_host_entry_points(tmp_path):
    if not os.path.exists(N.LIB_PATH):
        from long_context_tsa_b200 import build

        build.build()
    src = tmp_path / "abi.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(N.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-o", str(exe), "-L", libdir, "-l:libtsa.so", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.strip() == "ok"
