"""The boundary from plain C: include/spa.h compiles as C99 with every
warning an error, a C program links libspa.so and sees the validation
clauses (no device is touched)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c_and_library_links(tmp_path):
    from sparse_paged_attention_build_b200 import build
    build.build()
    pkg = os.path.join(ROOT, "sparse_paged_attention_build_b200")
    exe = str(tmp_path / "abi_from_c")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_from_c.c"),
                           "-L", pkg, "-lspa", "-Wl,-rpath," + pkg, "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip().endswith("ok")
