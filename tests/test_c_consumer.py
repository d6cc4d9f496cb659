"""The boundary is a plain C ABI: include/fa.h compiles as strict C99 (and C++),
and a C program links against libfa_sm100.so and calls it.  The program only
makes calls that the library rejects during argument validation, plus
fa_version, so it never touches a device (it runs the same on machines with and
without a GPU)."""
import os
import shutil
import subprocess

import pytest

from exact_tiled_attention_40_b200 import fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include "fa.h"

int main(void) {
  int bad = 0;
  /* negative batch: FA_ERR_INVALID_ARG before any device call */
  if (fa_fwd(0, 0, 0, 0, 0, -1, 1, 1, 8, 8, 128, 0.1f, 0, 0) != FA_ERR_INVALID_ARG) bad |= 1;
  /* unsupported head dimension */
  if (fa_decode_paged(0, 0, 0, 0, 0, 0, 1, 8, 2, 96, 16, 0.1f, 0, 4, 10, 0) != FA_ERR_UNSUPPORTED)
    bad |= 2;
  /* FP8 forward: D = 64 is not supported (checked after the pointers) */
  {
    void* p = (void*)0x10000;
    if (fa_fwd_fp8(p, p, p, (float*)p, (float*)p, (float*)p, p, 0, 1, 2, 1, 8, 8, 64, 0.1f, 0,
                   0) != FA_ERR_UNSUPPORTED)
      bad |= 4;
  }
  /* backward: null lse */
  if (fa_bwd((void*)0x10000, (void*)0x10000, (void*)0x10000, (void*)0x10000, 0,
             (void*)0x10000, (void*)0x10000, (void*)0x10000, (void*)0x10000, (float*)0x10000,
             1, 2, 1, 8, 8, 128, 0.1f, 0, 0) != FA_ERR_INVALID_ARG)
    bad |= 8;
  /* merge: negative row count */
  if (fa_merge_partials(0, 0, 0, 0, 0, -1LL, 128, 0, 0) != FA_ERR_INVALID_ARG) bad |= 16;
  printf("version %d, checks %s, last error: %s\n", fa_version(), bad ? "FAILED" : "ok",
         fa_last_error_string());
  return bad;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_is_c99_and_a_c_program_links_and_calls_the_library(tmp_path):
    lib_dir = os.path.dirname(fa.LIB_PATH)
    if not os.path.exists(fa.LIB_PATH):
        pytest.skip("library not built")
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I",
           os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", lib_dir,
           "-lfa_sm100", f"-Wl,-rpath,{lib_dir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "checks ok" in r.stdout


@pytest.mark.skipif(shutil.which("g++") is None, reason="no C++ compiler")
def test_header_compiles_as_cpp(tmp_path):
    src = tmp_path / "consumer.cpp"
    src.write_text('#include "fa.h"\nint main() { return fa_version() > 0 ? 0 : 1; }\n')
    r = subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-I",
                        os.path.join(ROOT, "include"), "-fsyntax-only", str(src)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
