"""The boundary is a C ABI: include/hsl.h must compile as strict C99, and a C
program linked against libhsl.so must see the documented host-side statuses.
Only argument checks run here (no device call is reached), so no GPU is needed."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(ROOT, "sparse_rank_linear_03_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "hsl.h"

static int fails = 0;
#define EXPECT(cond) do { if (!(cond)) { printf("FAIL %s:%d %s\n", __FILE__, __LINE__, #cond); ++fails; } } while (0)

int main(void) {
  hsl_handle h = NULL;
  hsl_group g = NULL;
  int64_t nnz = -1;
  EXPECT(hsl_create(0, 8, 2, HSL_FMT_CSR, HSL_F32, &h) == HSL_ERR_INVALID_ARG && h == NULL);
  EXPECT(strlen(hsl_last_message()) > 0);
  EXPECT(hsl_create(8, 6, 2, HSL_FMT_NM24, HSL_BF16, &h) == HSL_ERR_UNSUPPORTED);
  EXPECT(hsl_create(8, 8, 300, HSL_FMT_CSR, HSL_BF16, &h) == HSL_ERR_UNSUPPORTED);
  EXPECT(hsl_create(8, 8, 2, HSL_FMT_CSR, HSL_BF16, NULL) == HSL_ERR_INVALID_ARG);
  EXPECT(hsl_create(8, 8, 2, HSL_FMT_CSR, HSL_BF16, &h) == HSL_OK && h != NULL);
  EXPECT(hsl_split_topk(h, NULL, HSL_BF16, 0.5, NULL, NULL) == HSL_ERR_INVALID_ARG);
  EXPECT(hsl_apply(h, (const void*)16, (void*)16, 1, NULL) == HSL_ERR_NOT_READY);
  EXPECT(hsl_apply(h, (const void*)16, (void*)16, 0, NULL) == HSL_OK);
  EXPECT(hsl_get_nnz(h, &nnz) == HSL_OK && nnz == 0);
  EXPECT(hsl_group_create(&h, 1, &g, NULL) == HSL_ERR_NOT_READY && g == NULL);
  EXPECT(hsl_check(h, NULL) == HSL_OK);
  EXPECT(hsl_destroy(h) == HSL_OK);
  EXPECT(hsl_destroy(NULL) == HSL_OK);
  EXPECT(strcmp(hsl_status_str(HSL_ERR_TIMEOUT), hsl_status_str(HSL_OK)) != 0);
  printf("%s\n", fails ? "failed" : "ok");
  return fails != 0;
}
"""


@pytest.fixture(scope="module")
def cc():
    exe = shutil.which("gcc") or shutil.which("cc")
    if exe is None:
        pytest.skip("no C compiler")
    if not os.path.exists(os.path.join(LIBDIR, "libhsl.so")):
        pytest.skip("libhsl.so not built")
    return exe


def test_header_is_strict_c99(cc, tmp_path):
    src = tmp_path / "only_header.c"
    src.write_text('#include "hsl.h"\nint main(void) { return HSL_OK; }\n')
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", INCLUDE, "-c", str(src), "-o", str(tmp_path / "o.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_c_program_sees_documented_statuses(cc, tmp_path):
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", INCLUDE, str(src),
                        "-L", LIBDIR, "-lhsl", "-Wl,-rpath," + LIBDIR, "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.strip().endswith("ok")
