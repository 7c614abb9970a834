"""The C example of the README compiles against include/moe.h (gcc, C11,
warnings as errors), so the documented calls keep matching the header."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")


def test_readme_c_example_compiles(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not found")
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```c\n(.*?)```", text, re.S)
    assert blocks, "the README has a C example"
    src = tmp_path / "example.c"
    src.write_text("\n".join(blocks))
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-c",
                        "-I", os.path.join(ROOT, "include"), "-I", CUDA_INC, str(src),
                        "-o", str(tmp_path / "example.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
