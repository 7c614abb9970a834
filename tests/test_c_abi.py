"""The boundary seen from C: include/moe.h compiles as C99 (no C++ in the
header), and a C program links against libmoe.so and calls the host-only
entry points (no GPU needed: shape checks, status strings, null handles)."""
import os
import shutil
import subprocess

import pytest

from mixture_experts_layer_39_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "moe.h"

int main(void) {
  moe_shape_t s;
  int64_t rows = 0;
  memset(&s, 0, sizeof(s));
  s.T = 16384; s.d_model = 2048; s.d_ff = 1024; s.n_experts = 8; s.top_k = 4;
  s.dtype = MOE_DTYPE_BF16;
  if (moe_max_rows(&s, &rows) != MOE_OK) return 1;
  if (rows != 16384LL * 4 + 31 * 8) return 2;
  s.d_model = 200;                                   /* not a multiple of 128 */
  if (moe_max_rows(&s, &rows) != MOE_ERR_UNSUPPORTED) return 3;
  if (moe_destroy(NULL) != MOE_ERR_INVALID_ARG) return 4;
  if (moe_create(NULL, 0) != MOE_ERR_INVALID_ARG) return 5;
  if (moe_status_string(MOE_OK) == NULL) return 6;
  printf("%s|%s\n", moe_status_string(MOE_ERR_UNSUPPORTED), moe_status_string(12345));
  return 0;
}
"""


@pytest.fixture(scope="module")
def libdir():
    if not os.path.exists(_lib.LIB_PATH):
        from mixture_experts_layer_39_b200 import build
        build.build()
    return os.path.dirname(_lib.LIB_PATH)


def test_header_is_plain_c(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "h.c"
    src.write_text('#include "moe.h"\nint main(void) { return 0; }\n')
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I",
                        os.path.join(ROOT, "include"), "-c", str(src), "-o",
                        str(tmp_path / "h.o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_c_program_links_and_calls_host_entry_points(tmp_path, libdir):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        str(src), "-L", libdir, "-lmoe", "-Wl,-rpath," + libdir, "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, (run.returncode, run.stderr)
    unsupported, unknown = run.stdout.strip().split("|")
    assert unsupported and "unknown" in unknown


def test_readme_c_example_compiles(tmp_path):
    """The C example in the README is code against the real header."""
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    import re
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```c\n(.*?)```", text, re.S)
    assert blocks
    src = tmp_path / "example.c"
    src.write_text(blocks[0])
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        "-c", str(src), "-o", str(tmp_path / "example.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
