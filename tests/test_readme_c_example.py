"""CPU: the C example in README.md compiles against include/nvfp4ws.h (syntax and types only;
nothing runs)."""

import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")


@pytest.mark.skipif(shutil.which("gcc") is None or not os.path.isdir(CUDA_INC), reason="needs gcc and CUDA headers")
def test_readme_c_example_compiles(tmp_path):
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```c\n(.*?)```", text, flags=re.S)
    assert blocks, "README has no C example"
    src = tmp_path / "example.c"
    src.write_text(blocks[0])
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-fsyntax-only", "-I", os.path.join(ROOT, "include"),
                        "-I", CUDA_INC, str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
