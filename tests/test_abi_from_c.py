"""The C ABI from C: include/moe.h compiles as strict C99 (gcc, -Wall -Wextra
-Werror -pedantic) and a C program links libmoe_b200.so and gets its argument
errors, with no GPU present."""

import os
import shutil
import subprocess

import pytest

from sparse_moe_transformer_gemm_b200 import build as moe_build
from sparse_moe_transformer_gemm_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_header_compiles_as_c99_and_the_library_links_from_c(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    moe_build.build()
    libdir = os.path.dirname(moe.LIB_PATH)
    exe = str(tmp_path / "abi_c_check")
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    os.path.join(ROOT, "tests", "abi_c_check.c"), "-o", exe, "-L" + libdir,
                    "-l:" + os.path.basename(moe.LIB_PATH), "-Wl,-rpath," + libdir],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
