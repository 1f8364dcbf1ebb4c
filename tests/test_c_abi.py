"""The C ABI from plain C99, with no Python in the process that calls it:
- tests/c/abi_host_check.c, compiled with gcc against include/zero.h (-std=c99 -pedantic
  -Werror) and linked to libzero_b200.so, runs the host-only calls (layout, tables,
  counters, status strings) and checks closed forms;
- tests/c/abi_device_check.c (GPU) allocates with the CUDA runtime, runs three fused
  steps and writes inputs and outputs, which must equal the oracle's bit for bit."""
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


@pytest.mark.gpu
@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c_program_runs_the_step_and_matches_the_oracle(tmp_path):
    """tests/c/abi_device_check.c allocates with the CUDA runtime and runs three fused
    steps through the C ABI alone; its results equal the oracle's bit for bit."""
    import numpy as np
    import oracle
    from oracle.layout import make_layout
    build.build()
    exe, out = tmp_path / "abi_device_check", tmp_path / "out.bin"
    lib_dir = os.path.dirname(_abi.LIB_PATH)
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c", "abi_device_check.c"),
                    _abi.LIB_PATH, f"-Wl,-rpath,{lib_dir}", "-L", os.path.join(cuda, "lib64"), "-lcudart",
                    f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}", "-o", str(exe)], check=True)
    res = subprocess.run([str(exe), str(out)], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0 and res.stdout.strip() == "ok", res.stdout + res.stderr
    raw = out.read_bytes()
    N, P = np.frombuffer(raw[:16], np.int64)
    o = 16
    g = np.frombuffer(raw[o:o + 2 * N * P], np.uint16).reshape(N, P)
    o += 2 * N * P
    f32 = lambda k: np.frombuffer(raw[o + 4 * P * k:o + 4 * P * (k + 1)], np.float32)
    master0, master, m, v = f32(0), f32(1), f32(2), f32(3)
    p16 = np.frombuffer(raw[o + 16 * P:o + 18 * P], np.uint16)
    lay = make_layout([70001, 4099], 3, 7001, 8)
    assert lay.padded == P
    zeros = np.zeros(P, np.float32)
    ref = oracle.run_steps(lay, 2, np.ascontiguousarray(g), master0, zeros, zeros,
                           oracle.Hyper(1e-3, 0.9, 0.999, 1e-8, 0.01, 1024.0), 3)
    for name, got, want in (("master", master, ref.master), ("m", m, ref.m), ("v", v, ref.v),
                            ("p16", p16, ref.p16_full)):
        assert np.array_equal(np.ascontiguousarray(got).view(np.uint8), np.ascontiguousarray(want).view(np.uint8)), name
