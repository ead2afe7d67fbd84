"""The boundary is usable from plain C: include/velox.h compiles as C99 with
-pedantic -Werror, and a C program links libvelox.so and calls it.

Only calls that return before touching a device are made (host queries and
argument errors), so the test is safe on any machine.
"""

import os
import shutil
import subprocess

import pytest

from conftest import ROOT

C_SOURCE = r"""
#include <stdio.h>
#include <string.h>
#include "velox.h"

int main(void) {
  size_t ws = 0, mw = 0;
  if (velox_abi_version() != 104) return 1;
  if (velox_workspace_size(40, 48, 2256, 128, &ws) != VELOX_OK || ws == 0) return 2;
  if (velox_multiwarp_workspace_size(60, 4, 32, 48, &mw) != VELOX_OK) return 3;
  if (mw != (size_t)4 * 60 * 4 * 32 * 48) return 4;
  /* null tensors: refused on the host, nothing launched */
  if (velox_block_sparse_attn(NULL, NULL, NULL, NULL, NULL, NULL, 0, 1, 1, 1, 128, 128, 0.0f,
                              NULL, NULL, NULL, NULL) != VELOX_ERR_INVALID_ARG) return 5;
  if (velox_wait_selftest(0, NULL, NULL, NULL) != VELOX_ERR_INVALID_ARG) return 6;
  if (strcmp(velox_status_string(VELOX_OK), "ok") != 0) return 7;
  printf("%d %zu\n", velox_abi_version(), ws);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c99_program_links_and_calls_the_library(tmp_path):
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "velox_build", os.path.join(ROOT, "routed_block_sparse_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    lib = mod.build()
    src = tmp_path / "consumer.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(lib)
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-I", os.path.join(ROOT, "include"), str(src), "-L", libdir, "-lvelox",
                         f"-Wl,-rpath,{libdir}", "-o", str(exe)], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    assert run.stdout.split()[0] == "104"
