"""The boundary is a C ABI: include/vsa.h must compile as plain C (not C++),
and a C program must link against libvsa.so and call it. Only host-side entry
points are called (no GPU here): workspace size and layout, configuration
validation, status strings and the NULL-argument checks.
"""
import os
import shutil
import subprocess

import pytest

from trainable_block_sparse_cube_b200 import build as vsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "vsa.h"

int main(void) {
  vsa_config cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.B = 1; cfg.heads = 12; cfg.T = 16; cfg.H = 48; cfg.W = 80; cfg.D = 128; cfg.topk = 32;
  size_t bytes = vsa_workspace_bytes(&cfg);
  vsa_workspace_layout_t lay;
  vsa_status s = vsa_workspace_layout(&cfg, &lay);
  if (s != VSA_OK || bytes == 0 || lay.total != bytes) return 1;
  cfg.T = 6;  /* not a multiple of 4 */
  if (vsa_workspace_bytes(&cfg) != 0 || vsa_workspace_layout(&cfg, &lay) != VSA_ERR_SHAPE) return 2;
  if (vsa_run(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL) != VSA_ERR_INVALID_ARG) return 3;
  if (vsa_check(NULL) != VSA_ERR_INVALID_ARG) return 4;
  vsa_plan_destroy(NULL);
  printf("%s %zu\n", vsa_status_string(VSA_ERR_TIMEOUT), bytes);
  return 0;
}
"""


@pytest.fixture(scope="module")
def lib_dir():
    vsa_build.build()
    return os.path.join(ROOT, "trainable_block_sparse_cube_b200")


def test_header_compiles_as_c_and_links(tmp_path, lib_dir):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "main.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "main"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"), str(src),
                    "-L", lib_dir, "-lvsa", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stderr)
    name, nbytes = r.stdout.split()
    assert name == "VSA_ERR_TIMEOUT" and int(nbytes) > 0
