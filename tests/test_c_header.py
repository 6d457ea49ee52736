"""The C ABI from C: include/hadq.h compiles as C99 and a program linked
against libhadq.so runs the host-only entry points (no GPU needed)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB_DIR = os.path.join(ROOT, "hadamard_rotation_outlier_b200")

C_SOURCE = r"""
#include <stdio.h>
#include <string.h>
#include "hadq.h"

static int fails = 0;
#define CHECK(c) do { if (!(c)) { printf("FAILED: %s (line %d)\n", #c, __LINE__); fails++; } } while (0)

int main(void) {
  CHECK(hadq_version() > 0);
  CHECK(strlen(hadq_status_str(HADQ_ERR_INVALID_ARG)) > 0);

  hadq_path path = HADQ_PATH_NONE;
  CHECK(hadq_plan(0, 524288, 128, -1, 8, -1, 0, 1, &path) == HADQ_OK);
  CHECK(path == HADQ_PATH_CHUNK_MMA);
  CHECK(hadq_plan(0, 16384, 4096, -1, 4, -1, 1, 1, &path) == HADQ_OK);
  CHECK(path == HADQ_PATH_H4096_TC);
  CHECK(hadq_plan(0, 4, 96, 64, 8, -1, 0, 1, &path) == HADQ_ERR_INVALID_ARG);
  CHECK(strlen(hadq_last_error()) > 0);

  int32_t variant = -1;
  CHECK(hadq_kron_plan(0, 8192, 20, 256, 4, 128, 1, &variant) == HADQ_OK);
  CHECK(variant == HADQ_KRON_MMA);

  size_t ws = 0;
  CHECK(hadq_kv_decode_workspace_size(1, 32, 8, 131072, &ws) == HADQ_OK);
  CHECK(ws > 0);

  /* invalid sizes are rejected on the host, before any launch */
  const int64_t n0 = hadq_launch_count();
  CHECK(hadq_rotate_quantize(NULL, 4, 128, 48, NULL, 4, -1, NULL, NULL, NULL, NULL) == HADQ_ERR_INVALID_ARG);
  CHECK(hadq_rotate_quantize(NULL, 0, 128, 128, NULL, 4, 128, NULL, NULL, NULL, NULL) == HADQ_OK);
  CHECK(hadq_launch_count() == n0);

  printf(fails ? "c-abi: %d failures\n" : "c-abi ok\n", fails);
  return fails != 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c99_and_links(tmp_path):
    lib = os.path.join(LIB_DIR, "libhadq.so")
    if not os.path.exists(lib):
        pytest.skip("libhadq.so is not built")
    src = tmp_path / "abi.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "abi"
    cmd = ["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"), str(src),
           "-o", str(exe), "-L", LIB_DIR, "-lhadq", f"-Wl,-rpath,{LIB_DIR}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c-abi ok" in r.stdout
