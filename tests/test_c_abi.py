"""The C ABI from plain C99: tests/c/abi_host_check.c, compiled with gcc against
include/zero.h (-std=c99 -pedantic -Werror) and linked to libzero_b200.so, runs the
host-only calls (layout, tables, counters, status strings) and checks closed forms."""
import os
import shutil
import subprocess

import pytest

from zero_sharded_optimizer_ring_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_header_compiles_as_c99_and_host_calls_work(tmp_path):
    build.build()
    exe = tmp_path / "abi_host_check"
    lib_dir = os.path.dirname(_abi.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host_check.c"), _abi.LIB_PATH,
                    f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
