"""The C ABI from C: include/qlinear.h compiles as strict C99 (and as C++17)
without warnings, and a C program links against libqlinear.so and gets the
host-side answers (ABI version, status strings, size queries, argument
checks) without a GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(ROOT, "bit_quantized_linear_block_b200")

PROGRAM = r"""
#include <stdio.h>
#include "qlinear.h"

int main(void) {
  ql_weights w = {0};
  ql_tdc_params prm = {0.05f, 0.1f, 0.3f, 3, 8.0f, 1.0f};
  w.fmt = QL_W_NVFP4;
  w.N = 1920;
  w.K = 1920;
  printf("%d\n", qlinear_abi_version());
  printf("%s\n", qlinear_status_string(QL_ERR_UNSUPPORTED_SHAPE));
  printf("%zu\n", qlinear_sf_bytes(300, 640));
  printf("%d\n", (int)qlinear_forward(NULL, 10, &w, QL_ROUTE_NVFP4, NULL, NULL, 0, NULL));
  printf("%d\n", (int)qlinear_tdc_skip(NULL, -1, NULL, NULL, NULL, &prm, NULL, NULL));
  printf("%d\n", (int)qlinear_route_from_sums(NULL, 0.05f, NULL, NULL, NULL));
  return 0;
}
"""


@pytest.fixture(scope="module")
def compilers():
    if shutil.which("gcc") is None or shutil.which("g++") is None:
        pytest.skip("gcc/g++ not available")
    if not os.path.exists(os.path.join(LIBDIR, "libqlinear.so")):
        pytest.fail("libqlinear.so is missing: run the build first")


def test_header_is_strict_c99_and_cpp17(compilers, tmp_path):
    src = tmp_path / "hdr.c"
    src.write_text('#include "qlinear.h"\nint main(void) { return qlinear_abi_version() > 0 ? 0 : 1; }\n')
    for cmd in (["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only"],
                ["g++", "-std=c++17", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only", "-x", "c++"]):
        r = subprocess.run(cmd + ["-I", INCLUDE, str(src)], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_c_program_links_and_gets_host_answers(compilers, tmp_path):
    src, exe = tmp_path / "prog.c", tmp_path / "prog"
    src.write_text(PROGRAM)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", INCLUDE, str(src), "-L", LIBDIR, "-lqlinear",
                        f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    with open(os.path.join(INCLUDE, "qlinear.h")) as f:
        abi = next(int(ln.split()[2]) for ln in f if ln.startswith("#define QLINEAR_ABI_VERSION"))
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    lines = out.stdout.split("\n")
    assert lines[0] == str(abi)
    assert lines[1] == "unsupported shape"
    assert lines[2] == str(384 * (640 // 16))          # rows padded to 128: 384 x 40 scale bytes
    assert lines[3:6] == ["1", "1", "1"]               # QL_ERR_INVALID_ARG, before any CUDA call
