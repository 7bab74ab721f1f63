"""The host block manager under the address and undefined-behaviour sanitizers.

tests/bm_fuzz.c drives random histories (requests with repeating prompts,
decode appends, batched decode steps, forks, frees, an exhausted pool) through
pa_bm_* and checks the manager's invariants after every operation.  The block
manager is host code only, so it is compiled here from its source together
with the driver, with -fsanitize=address,undefined; any memory error or
undefined behaviour aborts the run.  CPU only.
"""

import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "paged_kv_cache_382_b200", "csrc", "block_manager.cpp")
DRIVER = os.path.join(ROOT, "tests", "bm_fuzz.c")
SAN = ["-g", "-O1", "-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer"]


@pytest.fixture(scope="module")
def fuzz_binary(tmp_path_factory):
    if not (shutil.which("gcc") and shutil.which("g++")):
        pytest.skip("gcc / g++ not found")
    d = tmp_path_factory.mktemp("bm_fuzz")
    inc = os.path.join(ROOT, "include")
    steps = [["gcc", "-std=c99", "-Wall", "-Werror", *SAN, "-I", inc, "-c", DRIVER, "-o", str(d / "f.o")],
             ["g++", "-std=c++17", *SAN, "-I", inc, "-c", SRC, "-o", str(d / "bm.o")],
             ["g++", "-fsanitize=address,undefined", str(d / "f.o"), str(d / "bm.o"), "-o", str(d / "bm_fuzz")]]
    for cmd in steps:
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0 and "sanitize" in res.stderr and "cannot find" in res.stderr:
            pytest.skip("sanitizer runtime not available")
        assert res.returncode == 0, res.stderr
    return str(d / "bm_fuzz")


@pytest.mark.parametrize("seed", [1, 2, 3, 4])
def test_random_histories_keep_the_invariants_under_sanitizers(fuzz_binary, seed):
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0", UBSAN_OPTIONS="print_stacktrace=1")
    res = subprocess.run([fuzz_binary, str(seed), "2000", "-v"], capture_output=True, text=True, env=env,
                         timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
    # the histories reach the interesting paths
    hits, copies, full = (int(x) for x in re.findall(r"\d+", res.stdout)[-3:])
    assert hits > 0 and copies > 0 and full > 0
