"""The bounds-checking build runs the reduced-size GPU parity suite green.

libzero_b200_debug.so is the library compiled with ZERO_DEBUG: every kernel that walks the
segment table checks each located segment and tile against the table's length, the
tile's shard, the padded buffer and the launch's state buffers; a tile that fails is
skipped and ZERO_ERR_BOUNDS is recorded in the layout's error word (no trap).  The
parity suite calls zero_get_error after its steps, so a failed check fails the test, and
a skipped tile would also show up as a mismatch against the oracle.  This stands in for
a memory checker, which these tests cannot use.

The suite runs in a child process with ZERO_B200_DEBUG=1 (the binding then loads the
debug library); full-size cases are left out (they only repeat the same checks on more
tiles).
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

SUITE = ["test_gpu_parity.py", "test_gpu_pipeline.py", "test_gpu_rank_counts.py", "test_gpu_wire.py",
         "test_gpu_ranks.py", "test_gpu_zero3_schedule.py", "test_zz_no_alloc.py"]


def _env():
    return dict(os.environ, ZERO_B200_DEBUG="1")


def test_debug_build_is_the_library_loaded():
    code = ("import zero_sharded_optimizer_ring_b200 as zs; zs._abi.lib(); "
            "print(zs._abi.LIB_PATH)")
    r = subprocess.run([sys.executable, "-c", code], env=_env(), cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip().endswith("libzero_b200_debug.so"), r.stdout


def test_parity_suite_under_the_debug_build():
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider",
           "-k", "not full_size and not beyond_2_32 and not two_process and not process_per_rank",
           *[os.path.join(HERE, f) for f in SUITE]]
    r = subprocess.run(cmd, env=_env(), cwd=ROOT, capture_output=True, text=True, timeout=1500)
    tail = (r.stdout[-3000:] + "\n" + r.stderr[-2000:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and " failed" not in r.stdout, tail
