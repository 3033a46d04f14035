"""The C ABI from C: tests/c_abi_check.c compiles against include/kvq.h as C11
(gcc, -Wall -Werror), links libkvq.so and runs its host-only calls, no GPU."""
import os
import shutil
import subprocess

import pytest

import quantized_kv_cache_17_b200 as kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_kv_cache_17_b200 import build
    build.build()


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_header_is_c_and_host_calls_run_from_c(tmp_path):
    exe = tmp_path / "c_abi_check"
    libdir = os.path.dirname(kvq.LIB_PATH)
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", str(exe), "-L", libdir, "-l:libkvq.so",
           "-Wl,-rpath," + libdir]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, f"check {r.returncode} failed: {r.stdout} {r.stderr}"
    assert r.stdout.startswith("kvq")
