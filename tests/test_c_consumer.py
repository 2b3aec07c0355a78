"""The boundary is a C ABI: include/pi_ffn.h compiles as strict C99 with all
warnings as errors, and a plain C program links against libpi_ffn.so and
calls its host-side entry points (no device is touched: the calls below all
fail argument validation before any launch)."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "activation_sparse_decode_gemv_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "pi_ffn.h"

int main(void) {
  int bad = 0;
  for (int s = PI_OK; s <= PI_ERR_WORKSPACE; ++s) {
    const char *t = pi_status_string((pi_status)s);
    if (!t || !*t) bad = 1;
  }
  pi_ffn_desc d;
  memset(&d, 0, sizeof d);                 /* d_model = 0: invalid */
  pi_ffn_t h = NULL;
  if (pi_ffn_create(&d, &h) != PI_ERR_INVALID_ARG || h != NULL) bad = 2;
  size_t bytes = 0;
  if (pi_workspace_size(NULL, 1, 1, &bytes) != PI_ERR_INVALID_ARG) bad = 3;
  if (pi_decode_ffn(NULL, NULL, 1, NULL, NULL, NULL, 0u, NULL, 0, NULL) != PI_ERR_INVALID_ARG) bad = 4;
  if (pi_workspace_init(NULL, 16, NULL) != PI_ERR_INVALID_ARG) bad = 5;
  pi_ffn_destroy(NULL);
  printf("c consumer %s\n", bad ? "FAILED" : "ok");
  return bad;
}
"""


@pytest.fixture(scope="module")
def lib_dir():
    if not os.environ.get("PI_FFN_LIB"):
        from activation_sparse_decode_gemv_b200 import build
        build.build()
    return PKG


def test_header_is_strict_c99(tmp_path):
    src = tmp_path / "only_header.c"
    src.write_text('#include "pi_ffn.h"\nint pi_header_compiles(void) { return PI_OK; }\n')
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Wpedantic", "-Werror", "-fsyntax-only",
                           "-I", os.path.join(ROOT, "include"), str(src)])


def test_c_program_links_and_calls(tmp_path, lib_dir):
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-o", str(exe),
                           str(src), "-L", lib_dir, "-lpi_ffn", f"-Wl,-rpath,{lib_dir}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120,
                         env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert out.returncode == 0, out.stdout + out.stderr
    assert "c consumer ok" in out.stdout
