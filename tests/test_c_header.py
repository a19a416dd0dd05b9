"""The C ABI from C: include/qmoe.h compiles as C99 (no C++ or CUDA types in
the signatures) and a C program links libqmoe.so and calls its entry points.
Only argument-validation paths run, so no GPU is needed."""
import os
import shutil
import subprocess

import pytest

from quantized_top_routed_b200 import qmoe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = r"""
#include <stdio.h>
#include <string.h>
#include "qmoe.h"

int main(void) {
  int fails = 0;
  /* NULL-safe destroy and an empty error string */
  if (qmoe_destroy(NULL) != QMOE_OK) fails++;
  /* create rejects a NULL config before touching the device */
  qmoe_handle* h = (qmoe_handle*)1;
  if (qmoe_create(NULL, NULL, NULL, NULL, &h) != QMOE_ERR_INVALID) fails++;
  if (h != NULL) fails++;                       /* *out is cleared on failure */
  if (strlen(qmoe_last_error()) == 0) fails++;
  /* d not a multiple of 128 */
  qmoe_config c = {200, 8, 2, 256, 0, 16};
  float w[1] = {0.f};
  qmoe_expert ex[8];
  memset(ex, 0, sizeof(ex));
  if (qmoe_create(&c, w, NULL, ex, &h) != QMOE_ERR_INVALID) fails++;
  /* calls on a NULL handle */
  if (qmoe_forward(NULL, NULL, 4, NULL, NULL) != QMOE_ERR_INVALID) fails++;
  if (qmoe_check_error(NULL, NULL) != QMOE_ERR_INVALID) fails++;
  if (qmoe_launches_per_forward(NULL, 4) != 0) fails++;
  /* the no-allocation router validates sizes first */
  if (qmoe_route_topk_noalloc((const uint16_t*)16, (const float*)16, NULL, QMOE_ROUTE_STATIC_MAX_LOGITS, 256, 8, 2,
                              (int32_t*)16, (float*)16, NULL) != QMOE_ERR_INVALID) fails++;
  printf("fails=%d\n", fails);
  return fails;
}
"""


@pytest.fixture(scope="module")
def lib_path():
    qmoe.load()                                   # builds in-tree if needed
    return qmoe._build.LIB


def test_header_compiles_as_c99_and_entry_points_work_from_c(tmp_path, lib_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(C_SRC)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib_path)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                        str(exe), f"-L{libdir}", "-l:libqmoe.so", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "fails=0" in run.stdout
