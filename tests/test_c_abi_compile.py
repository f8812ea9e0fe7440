"""The C ABI from C: include/fp8lin.h compiles as strict C99 (and as C++17),
and a C program links against libfp8lin.so and calls the entry points that
need no GPU (version, ring size, argument validation, the GEMM tile plan)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INC = os.path.join(ROOT, "include")
LIBDIR = os.path.join(ROOT, "fp8_delayed_scaling_03_b200", "lib")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "fp8lin.h"

int main(void) {
  fp8_mm_args a;
  fp8_mm_plan_info info;
  memset(&a, 0, sizeof(a));
  a.m = 2048; a.n = 1024; a.k = 1024;
  a.a = (const uint8_t*)0x100000; a.lda = 1024; a.fmt_a = FP8_E4M3; a.a_major = FP8_K_MAJOR;
  a.b = (const uint8_t*)0x200000; a.ldb = 1024; a.fmt_b = FP8_E4M3; a.b_major = FP8_K_MAJOR;
  a.scale_a = (const float*)0x300000; a.scale_b = (const float*)0x300010;
  a.d = (void*)0x400000; a.ldd = 1024;
  int s = fp8_mm_plan(&a, NULL, 148, &info);
  printf("%s|%d|%d|%lld|%d|%zu|%d|%d\n", fp8_version(), s, info.tile_cfg, (long long)info.tiles, info.units,
         fp8_ring_bytes(16), fp8_ring_init(NULL, 16, NULL), fp8_mm(NULL, NULL));
  return 0;
}
"""


@pytest.fixture(scope="module")
def lib():
    import fp8_delayed_scaling_03_b200  # noqa: F401  (the conftest built it; importing checks it loads)
    if not shutil.which("gcc"):
        pytest.skip("no C compiler")
    return LIBDIR


def test_header_is_strict_c99_and_cxx17(lib, tmp_path):
    src = tmp_path / "t.c"
    src.write_text(PROGRAM)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INC, "-fsyntax-only",
                    str(src)], check=True)
    if shutil.which("g++"):
        subprocess.run(["g++", "-std=c++17", "-Wall", "-Werror", "-I", INC, "-x", "c++", "-fsyntax-only", str(src)],
                       check=True)


def test_c_program_links_and_runs(lib, tmp_path):
    src = tmp_path / "t.c"
    exe = tmp_path / "t"
    src.write_text(PROGRAM)
    subprocess.run(["gcc", "-std=c99", "-I", INC, str(src), "-L", lib, "-lfp8lin", f"-Wl,-rpath,{lib}", "-o",
                    str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.strip()
    version, status, cfg, tiles, units, ring_bytes, init_null, mm_null = out.split("|")
    assert "sm_100a" in version
    assert (status, cfg, tiles, units) == ("0", "1", "128", "128")   # 128x128 tiles, one per SM
    assert ring_bytes == str((16 + 4) * 4)
    assert init_null == mm_null == "-1"                              # FP8_ERR_INVALID_ARG, nothing launched
