"""The boundary is a C ABI: a plain C99 program (tests/c_consumer.c), compiled
with gcc -std=c99 -pedantic -Werror against include/pa.h and linked to
libpa.so, calls the host-side entry points and checks their results.  No GPU."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_against_the_header_and_library(tmp_path):
    from paged_kv_cache_382_b200 import build

    build.build()
    libdir = os.path.join(ROOT, "paged_kv_cache_382_b200")
    exe = str(tmp_path / "c_consumer")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_consumer.c"), "-o", exe, f"-L{libdir}", "-l:libpa.so",
           f"-Wl,-rpath,{libdir}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    assert "c consumer ok" in run.stdout
