"""The boundary from C: include/moe.h compiles as C99 with warnings as
errors, and a C program linked against libmoe.so calls its host-side entry
points (sizes, capacity, argument checks: no kernel is launched, no GPU is
needed)."""

import os
import shutil
import subprocess

import pytest

from mixture_experts_layer_51_b200 import moe as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "mixture_experts_layer_51_b200")

PROGRAM = r"""
#include <math.h>
#include <stdio.h>
#include "moe.h"

int main(void) {
  moe_ws_layout L;
  moe_graph* g = NULL;
  moe_pipeline* p = NULL;
  if (moe_abi_version() != MOE_ABI_VERSION) return 1;
  /* C = ceil(1.25 * 256 * 1 / 4) = 80; dropless below 0 */
  if (moe_capacity(256, 4, 1, 1.25) != 80) return 2;
  if (moe_max_permuted_rows(4096, 8, 2, 0.0) != 9216) return 3;
  if (moe_workspace_layout(8192, 4096, 14336, 8, 2, 0.0, MOE_BF16, MOE_SWIGLU, &L) != MOE_OK)
    return 4;
  if (moe_workspace_bytes(8192, 4096, 14336, 8, 2, 0.0, MOE_BF16, MOE_SWIGLU) != L.total) return 5;
  /* argument checks happen before anything touches the device */
  if (moe_forward(NULL, NULL, NULL, NULL, NULL, NULL, 16, 64, 64, 4, 5, 0.0, MOE_SWIGLU,
                  MOE_BF16, NULL, NULL, 0, NULL, NULL) != MOE_ERR_ARG) return 6;
  if (moe_forward_graph_create(NULL, NULL, NULL, NULL, NULL, NULL, 16, 64, 64, 4, 2, 0.0,
                               MOE_SWIGLU, MOE_BF16, NULL, NULL, NULL, 0, &g) != MOE_ERR_ARG)
    return 7;
  if (g != NULL || moe_forward_graph_destroy(NULL) != MOE_OK) return 8;
  if (moe_pipeline_create(MOE_PIPELINE_MAX_DEPTH + 1, &p) != MOE_ERR_ARG) return 9;
  if (moe_expert_choice_tokens(100, 4, 2, 1.0) != 50) return 10;
  printf("%s|%s\n", moe_status_string(MOE_OK), moe_status_string(MOE_ERR_ARG));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c99_and_links(tmp_path):
    M.lib()  # the library is built (raises otherwise)
    src = tmp_path / "abi_check.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
           "-L", PKG, "-lmoe", "-Wl,-rpath," + PKG, "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    ok, arg = run.stdout.strip().split("|")
    assert ok and arg and ok != arg
