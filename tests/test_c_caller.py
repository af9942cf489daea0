"""The boundary from plain C (CPU only): ``include/qlinear.h`` compiles as C99
with warnings as errors, a C program links ``libqlinear.so`` directly (no
Python, no torch), and the host-side argument checks return their documented
status codes before anything touches a device."""
import os
import shutil
import subprocess

import pytest

from fp8_linear_layers_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = r"""
#include <stdio.h>
#include <string.h>
#include "qlinear.h"

#define CHECK(expr, want)                                                   \
  do {                                                                      \
    ql_status got_ = (expr);                                                \
    if (got_ != (want)) {                                                   \
      printf("line %d: %s returned %d, expected %d\n", __LINE__, #expr,     \
             (int)got_, (int)(want));                                       \
      return 1;                                                             \
    }                                                                       \
  } while (0)

int main(void) {
  /* a 16-byte aligned address that the checks below never dereference */
  void* a = (void*)(uintptr_t)0x10000;
  const uint16_t* x = (const uint16_t*)a;
  uint16_t* y = (uint16_t*)a;
  const float* s = (const float*)a;

  if (strcmp(qlinear_status_string(QL_OK), qlinear_status_string(QL_ERR_CUDA)) == 0) return 2;
  if (strcmp(qlinear_status_string((ql_status)99), "unknown status") != 0) return 3;

  CHECK(qlinear_gemv((ql_scheme)7, x, a, s, 64, 64, y, NULL, NULL), QL_ERR_INVALID_ARG);
  CHECK(qlinear_gemv(QL_W8A8_INT8_ROW, NULL, a, s, 64, 64, y, NULL, NULL), QL_ERR_INVALID_ARG);
  CHECK(qlinear_gemv(QL_W8A8_INT8_ROW, x + 1, a, s, 64, 64, y, NULL, NULL), QL_ERR_MISALIGNED);
  CHECK(qlinear_gemv(QL_FP8_E4M3_BLOCK128, x, a, s, 64, 256, y, NULL, NULL),
        QL_ERR_UNSUPPORTED_SHAPE);
  CHECK(qlinear_gemv_weight_only(QL_FP8_E4M3_ROW, x, a, s, 64, 40, y, NULL),
        QL_ERR_UNSUPPORTED_SHAPE);
  CHECK(qlinear_gemv_weight_only(QL_FP8_E4M3_ROW, x, a, s, 64, 16400, y, NULL),
        QL_ERR_UNSUPPORTED_SHAPE);
  CHECK(qlinear_quantize_weight(QL_FP8_E4M3_BLOCK128, x, 100, 128, a, (float*)a, NULL),
        QL_ERR_UNSUPPORTED_SHAPE);
  CHECK(qlinear_quantize_act(QL_W8A8_INT8_ROW, x, -1, 64, a, (float*)a, NULL),
        QL_ERR_INVALID_ARG);
  CHECK(qlinear_gemm_small(QL_W8A8_INT8_ROW, x, a, s, 33, 64, 64, y, a, 1 << 20, NULL, NULL),
        QL_ERR_UNSUPPORTED_SHAPE);
  CHECK(qlinear_gemm_small_noalloc(QL_W8A8_INT8_ROW, x, a, s, 33, 64, 64, y, NULL),
        QL_ERR_UNSUPPORTED_SHAPE);
  CHECK(qlinear_gemm(QL_W8A8_INT8_ROW, a, s, a, s, 64, 64, 133152, y, NULL, 0, NULL, NULL),
        QL_ERR_UNSUPPORTED_SHAPE);
  /* M = 0 is a no-op that succeeds without a device */
  CHECK(qlinear_quantize_act(QL_W8A8_INT8_ROW, NULL, 0, 64, NULL, NULL, NULL), QL_OK);
  CHECK(qlinear_forward(QL_W8A8_INT8_ROW, NULL, NULL, NULL, 0, 64, 64, NULL, NULL, 0, NULL),
        QL_OK);
  printf("c caller ok\n");
  return 0;
}
"""


@pytest.fixture(scope="module")
def libdir():
    qbuild.build()
    return os.path.dirname(qbuild.LIB_PATH)


def test_header_compiles_as_c_and_links_from_c(tmp_path, libdir):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "caller.c"
    src.write_text(C_SRC)
    exe = tmp_path / "caller"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                        "-L", libdir, "-lqlinear", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "c caller ok" in run.stdout
