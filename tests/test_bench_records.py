"""bench.py's roofline bookkeeping on CPU: the algorithmic bytes per parameter, the
source hash that keeps a DRAM-traffic record tied to the kernel it was captured on, the
ncu CSV -> per-launch record conversion, and the rule that a record is used only for
the same sources and padded size.  Temporary files only; the committed records and
sources are not touched."""
import argparse
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from seeded_inputs.workloads import full_workloads, reduced_workloads  # noqa: E402


def test_bytes_per_param_follow_the_step():
    """2N gradient bytes + 12 state read + 12 state written + 2 fp16 written, plus one
    gather pass (2 + 2) for ZeRO-3."""
    wls = full_workloads()
    flat, llama = wls["flat1p3b_n4_zero1"], wls["llama3b_n8_zero3"]
    assert bench.fused_bytes_per_param(flat) == bench.ideal_bytes_per_param(flat) == 34
    assert bench.fused_bytes_per_param(llama) == 42 and bench.ideal_bytes_per_param(llama) == 46
    assert bench.throughput(1_000_000, 4, 2.0) == 1_000_000 * 4 / 0.002


@pytest.fixture
def sources(tmp_path, monkeypatch):
    a, b = tmp_path / "k.cu", tmp_path / "k.h"
    a.write_text("__global__ void k(float *x) { x[0] = 1.0f; }  // first\n")
    b.write_text("/* a header */\nint n = 3;\n")
    monkeypatch.setitem(bench.KERNEL_SOURCES, "probe", [str(a), str(b)])
    monkeypatch.setattr(bench, "PROFILE_DIR", str(tmp_path))
    return a, b


def test_hash_ignores_comments_and_spacing_but_not_code(sources):
    a, b = sources
    h0 = bench.kernel_source_hash("probe")
    a.write_text("__global__ void k(float *x)\n{\n    x[0] = 1.0f;   // reworded\n}\n")
    b.write_text("/* another\n   header comment */ int n = 3;\n")
    assert bench.kernel_source_hash("probe") == h0
    a.write_text("__global__ void k(float *x) { x[0] = 2.0f; }\n")
    assert bench.kernel_source_hash("probe") != h0


CSV = '''==PROF== Connected to process 1
"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"0","1","python","h","void probe_kernel<4>(Args)","1","7","(256, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","1,000,000"
"0","1","python","h","void probe_kernel<4>(Args)","1","7","(256, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","600,000"
"0","1","python","h","void probe_kernel<4>(Args)","1","7","(256, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","ns","2,000"
"1","1","python","h","other_kernel(int)","1","7","(256, 1, 1)","(1, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","5"
"2","1","python","h","void probe_kernel<4>(Args)","1","7","(256, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Mbyte","1.2"
"2","1","python","h","void probe_kernel<4>(Args)","1","7","(256, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","Kbyte","400"
"2","1","python","h","void probe_kernel<4>(Args)","1","7","(256, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","usecond","4"
'''


def _record(tmp_path, wl, kernel="probe_kernel", tag="probe"):
    csv = tmp_path / "capture.csv"
    csv.write_text(CSV)
    a = argparse.Namespace(record_traffic=str(csv), record_kernel=kernel, record_tag=tag, record_note="test")
    bench.record_traffic(a, wl)
    return json.load(open(bench.traffic_record_name(tag, wl.name)))


def test_record_is_the_mean_per_launch_of_the_named_kernel(sources, tmp_path, capsys):
    wl = reduced_workloads()["flat1p3b_n4_zero1"]
    rec = _record(tmp_path, wl)
    assert rec["launches"] == 2                                     # the other kernel's row is skipped
    assert rec["dram_bytes_read_per_launch"] == pytest.approx((1_000_000 + 1_200_000) / 2)
    assert rec["dram_bytes_write_per_launch"] == pytest.approx((600_000 + 400_000) / 2)
    assert rec["gpu_time_ms_per_launch"] == pytest.approx((0.002 + 0.004) / 2)
    assert rec["kernel_sources_sha256_16"] == bench.kernel_source_hash("probe")
    capsys.readouterr()


def test_record_is_used_only_for_the_same_sources_and_size(sources, tmp_path, capsys):
    wl = reduced_workloads()["flat1p3b_n4_zero1"]
    rec = _record(tmp_path, wl)
    P = rec["padded_params"]
    assert bench.profiled_traffic("probe", wl.name, P) == pytest.approx(1_100_000 + 500_000)
    assert bench.profiled_traffic("probe", wl.name, P + 128) is None         # another size
    assert bench.profiled_traffic("probe", "no_such_workload", P) is None    # no record
    a, _ = sources
    a.write_text(a.read_text() + "\n// a comment only\n")
    assert bench.profiled_traffic("probe", wl.name, P) is not None          # still the same kernel
    a.write_text("__global__ void k(float *x) { x[1] = 1.0f; }\n")
    assert bench.profiled_traffic("probe", wl.name, P) is None               # the kernel changed
    capsys.readouterr()


def test_record_without_both_dram_metrics_is_refused(sources, tmp_path):
    wl = reduced_workloads()["flat1p3b_n4_zero1"]
    with pytest.raises(SystemExit):
        _record(tmp_path, wl, kernel="other_kernel")


def test_default_run_times_both_roofline_workloads():
    """The plain `bench.py` run adds the Llama-shaped ZeRO-3 list to the flat headline in
    the same JSON line; variant runs and explicit --also choices do not."""
    a = bench.parse([])
    assert a.workload == bench.DEFAULT_WORKLOAD == "flat1p3b_n4_zero1"
    assert bench.also_workloads(a) == ["llama3b_n8_zero3"]
    for extra in (["--kernel", "1"], ["--wire-fp16"], ["--psi", "1048576"], ["--also", "none"],
                  ["--workload", "gpt2_small_n8_zero2"]):
        assert bench.also_workloads(bench.parse(extra)) == [], extra
    assert bench.also_workloads(bench.parse(["--also", "gpt2_small_n8_zero2"])) == [
        "gpt2_small_n8_zero2"]
