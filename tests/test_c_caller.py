"""The boundary from C: include/matq.h compiles as strict C11 and a C program links against
libmatq.so and gets the documented answers from the layout queries and the host-side argument
checks.  Every call here is a query or fails validation before any launch, so no GPU is needed.
"""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BUILD = os.path.join(ROOT, "tests", "_build", "c_caller")

PROGRAM = r"""
#include <stdint.h>
#include <stdio.h>
#include <string.h>
#include "matq.h"

#define CHECK(cond) do { if (!(cond)) { printf("FAILED line %d: %s\n", __LINE__, #cond); return 1; } } while (0)

int main(void) {
  void* fake = (void*)(uintptr_t)(1u << 20);   /* aligned, never dereferenced */
  int widths[3] = {3, 4, 8};
  float lambdas[3] = {1.0f, 1.0f, 1.0f};
  /* layout queries: r bits per weight when 16 | N */
  CHECK(matq_packed_bytes(16, 256, 2) == 16 * 256 * 2 / 8);
  CHECK(matq_packed_bytes(32, 512, 8) == 32 * 512);
  CHECK(matq_plane_count(4) == 3 && matq_plane_count(5) == 0);
  CHECK(matq_linear_workspace(1, 4096, 14336, 128) > 0);
  /* argument checks */
  CHECK(matq_pack(fake, 16, 256, 5, fake, 4096, 0) == MATQ_EINVAL_R);
  CHECK(matq_linear(fake, 1, 1000, fake, 8, fake, fake, 64, 4, 128, fake, MATQ_OUT_BF16, fake, 1u << 20, 0)
        == MATQ_EINVAL_SHAPE);
  CHECK(matq_linear(fake, 1, 256, fake, 4, fake, fake, 64, 8, 128, fake, MATQ_OUT_BF16, fake, 1u << 20, 0)
        == MATQ_ETRUNC);
  CHECK(matq_choose_codes(fake, 4, 128, fake, fake, 32, 3, widths, lambdas, MATQ_SLICE_TRUE_PREFIX, fake, 0)
        == MATQ_EINVAL_GROUP);
  lambdas[1] = -1.0f;
  CHECK(matq_choose_codes(fake, 4, 128, fake, fake, 64, 3, widths, lambdas, MATQ_SLICE_TRUE_PREFIX, fake, 0)
        == MATQ_EINVAL_ARG);
  CHECK(matq_silu_mul_gu(NULL, 1, 16, fake, 0) == MATQ_ENULL);
  CHECK(strlen(matq_strerror(MATQ_ECUDA)) > 0 && strlen(matq_strerror(MATQ_EINVAL_ARG)) > 0);
  printf("c caller ok\n");
  return 0;
}
"""


def test_c_program_links_and_gets_documented_answers():
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("needs gcc")
    from nested_bit_weight_msb_b200 import build
    build.build()
    libdir = os.path.join(ROOT, "nested_bit_weight_msb_b200")
    assert os.path.exists(os.path.join(libdir, "libmatq.so"))
    os.makedirs(BUILD, exist_ok=True)
    src = os.path.join(BUILD, "caller.c")
    exe = os.path.join(BUILD, "caller")
    with open(src, "w") as f:
        f.write(PROGRAM)
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    src, "-o", exe, "-L", libdir, "-l:libmatq.so", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "c caller ok" in out.stdout
