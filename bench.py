"""Benchmark of the fused sharded optimizer step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = zero_step over the whole workload: the ring reduce-scatter of every bucket
fused with the unscale + AdamW + fp16 update (and, for ZeRO-3, the all-gather of every
gather unit), with inputs resident in HBM.  With N GPUs every GPU runs its own replica of
the workload (the simulated ranks all live in one GPU's memory, so nothing is exchanged
between GPUs); the value is the total over GPUs, timed as the max over ranks.

--impl reference times the CPU oracle on a bounded sample of the same workload (rank 0
only; other ranks exit without work).
"""
import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "params updated/sec per zero_step and achieved HBM GB/s vs peak (1×B200)"
UNIT = "params/s"
DEFAULT_WORKLOAD = "flat1p3b_n4_zero1"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
PROFILE_DIR = os.path.join(ROOT, "profiles")
# the sources each recorded kernel is compiled from: a traffic record taken on other
# sources is stale
_CSRC = os.path.join(ROOT, "zero_sharded_optimizer_ring_b200", "csrc")
KERNEL_SOURCES = {tag: [os.path.join(_CSRC, f) for f in files] for tag, files in {
    "bulk_step": ("bulk_step.cu", "bulk_ptx.cuh", "device_common.cuh", "internal.h"),
    "tile_kernel": ("kernels.cu", "bulk_ptx.cuh", "device_common.cuh", "internal.h"),
    "copy_range": ("kernels.cu", "bulk_ptx.cuh", "device_common.cuh", "internal.h"),
}.items()}


def parse(argv=None):
    """The command line (argv: a list in place of sys.argv[1:])."""
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=4)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="--impl reference: oracle time budget of the whole run")
    ap.add_argument("--kernel", type=int, default=0, help="fused kernel: 0 auto, 1 register, 2 bulk")
    ap.add_argument("--wire-fp16", action="store_true",
                    help="partial sums travel the ring as fp16 (its own line; not the headline)")
    ap.add_argument("--dynamic", action="store_true",
                    help="time zero_step_dynamic (reduce-scatter, overflow check, update) instead of the fused step")
    ap.add_argument("--dynamic-commit", action="store_true",
                    help="time zero_step_dynamic_commit (one fused pass into a second state set, overflow "
                         "check, swap) instead of the fused step")
    ap.add_argument("--unfused", action="store_true",
                    help="time the standalone reduce-scatter, shard update and all-gather calls (its own JSON line)")
    ap.add_argument("--graph", action="store_true",
                    help="time steps launched one by one against the same steps replayed from CUDA graphs "
                         "(zero_step_device_scalars; its own JSON line)")
    ap.add_argument("--graph-steps", type=int, default=20, help="--graph: steps captured per graph")
    ap.add_argument("--zero3-passes", action="store_true",
                    help="time ZeRO-3's per-layer forward and backward gathers with 1-3 prefetch slots "
                         "against a simulated layer compute (its own JSON line)")
    ap.add_argument("--tokens", type=int, default=2048, help="--zero3-passes: tokens per rank")
    ap.add_argument("--zero3-configs", default="0:0:0,0:0:1,0:0:2,default,width",
                    help="--zero3-passes sweep: comma-separated carveout:gather_ctas:slots (carveout = how far "
                         "below the SM count the matmuls' cuBLAS SM-count target is set; gather_ctas = "
                         "zero_set_gather_ctas, 0 = default grid; slots 0 = the compute alone), or 'default' "
                         "(zero3_pass's own settings) or 'width' (those, with the gather width tuned per kind of "
                         "pass by schedule.GatherWidth)")
    ap.add_argument("--zero3-rounds", type=int, default=5, help="--zero3-passes: interleaved rounds of the sweep")
    ap.add_argument("--blas", default="", help="--zero3-passes: torch preferred BLAS library (cublas, cublaslt)")
    ap.add_argument("--overlap", action="store_true",
                    help="measure the bucket-pipelined step behind a simulated backward pass "
                         "(its own JSON line; not the headline)")
    ap.add_argument("--backward", default="generator", choices=["generator", "gemm"],
                    help="--overlap: the simulated backward. generator = the seeded generator's kernels "
                         "rewrite each bucket's gradients (ALU-bound); gemm = two bf16 GEMMs per bucket "
                         "(cuBLAS, 4 * tokens FLOPs per parameter; tensor-core bound)")
    ap.add_argument("--bwd-tokens", type=int, default=4096, help="--overlap --backward gemm: tokens per rank")
    ap.add_argument("--max-ctas", default="0",
                    help="cap on the fused kernel's CTAs (zero_set_max_ctas; 0 = one per SM, and for the "
                         "overlapped step the library's measured choice). With --overlap a comma-separated list, "
                         "one JSON line each")
    ap.add_argument("--bucket-group", default="auto",
                    help="--overlap: buckets per launch (zero_step_overlapped_grouped); auto = zero_step_overlapped "
                         "(small buckets coalesced); a comma-separated list, one JSON line each")
    ap.add_argument("--shrink", type=int, default=0,
                    help="divide every tensor of the workload by this factor (same structure, smaller: "
                         "small cases for profiler captures; not a bench line)")
    ap.add_argument("--also", default="auto",
                    help="workloads timed after the headline in the same run (comma-separated, or none); "
                         "auto = the Llama-shaped ZeRO-3 list after the default flat list")
    ap.add_argument("--record-traffic", default="",
                    help="host-only: read this ncu CSV (dram__bytes_read.sum, dram__bytes_write.sum, "
                         "gpu__time_duration.sum per launch) and write the per-launch traffic record of "
                         "--record-tag for --workload under profiles/")
    ap.add_argument("--record-kernel", default="bulk_step_kernel", help="--record-traffic: kernel name regex")
    ap.add_argument("--record-tag", default="bulk_step", help="--record-traffic: record name prefix")
    ap.add_argument("--record-note", default="", help="--record-traffic: how the capture was taken")
    ap.add_argument("--ranks", type=int, default=0,
                    help="run the workload with this many simulated ranks (rank-count studies; not a bench line)")
    ap.add_argument("--psi", type=int, default=0,
                    help="flat workloads only: run the same shape with this many parameters "
                         "(small cases for profiler captures; not a bench line)")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    return a


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def max_over_ranks(x, world, device):
    """The largest of the ranks' values (timing: the slowest rank defines the step)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(psi, world, ms):
    """Whole-job parameters per second: every rank updates its own replica of psi."""
    return psi * world / (ms / 1e3)


def ideal_bytes_per_param(wl):
    # grads 2N read; master, m, v read + write 24; fp16 write 2; ZeRO-3 gather 2 + 2
    return 2 * wl.n_ranks + 24 + 2 + (4 if wl.stage == 3 else 0)


def fused_bytes_per_param(wl):
    return 2 * wl.n_ranks + 24 + 2


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        return float(json.load(open(p))["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(kernel_tag):
    """Hash of the kernel's sources with comments and blank space removed, so that a
    traffic record stays valid across comment-only edits."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel_tag]:
        text = open(f).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def traffic_record_name(kernel_tag, workload):
    return os.path.join(PROFILE_DIR, f"{kernel_tag}_{workload}.json")


def profiled_traffic(kernel_tag, workload, padded):
    """DRAM bytes (read + write) per launch of a kernel on a workload, from the record
    `--record-traffic` wrote for a full-size capture of the same launch configuration
    on the current kernel sources; None when there is no such record."""
    try:
        rec = json.load(open(traffic_record_name(kernel_tag, workload)))
    except (OSError, ValueError):
        return None
    if rec.get("kernel_sources_sha256_16") != kernel_source_hash(kernel_tag) or rec.get("padded_params") != padded:
        return None
    return rec["dram_bytes_read_per_launch"] + rec["dram_bytes_write_per_launch"]


_NCU_UNITS = {"byte": 1.0, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "tbyte": 1e12,
              "ns": 1e-9, "us": 1e-6, "ms": 1e-3, "s": 1.0,
              "nsecond": 1e-9, "usecond": 1e-6, "msecond": 1e-3, "second": 1.0}


def record_traffic(a, wl):
    """Turn an ncu CSV capture (metrics dram__bytes_read.sum, dram__bytes_write.sum,
    gpu__time_duration.sum of the launches of one kernel) into the per-launch record
    profiled_traffic() reads.  Host-only; no GPU needed."""
    import csv
    rows = list(csv.reader(l for l in open(a.record_traffic) if l.startswith('"')))
    head, body = rows[0], rows[1:]
    col = {k: head.index(k) for k in ("ID", "Kernel Name", "Metric Name", "Metric Unit", "Metric Value")}
    launches = {}
    for r in body:
        if not re.search(a.record_kernel, r[col["Kernel Name"]]):
            continue
        unit = _NCU_UNITS.get(r[col["Metric Unit"]].strip().lower(), 1.0)
        val = float(r[col["Metric Value"]].replace(",", "")) * unit
        d = launches.setdefault(r[col["ID"]], {"kernel": r[col["Kernel Name"]]})
        d[r[col["Metric Name"]]] = val
    got = [d for d in launches.values() if "dram__bytes_read.sum" in d and "dram__bytes_write.sum" in d]
    if not got:
        raise SystemExit(f"no launch of {a.record_kernel!r} with both DRAM metrics in {a.record_traffic}")
    import zero_sharded_optimizer_ring_b200 as zs      # host-only partitioner: the padded size
    P = zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units)).padded
    n = len(got)
    rec = {"kernel": got[0]["kernel"], "workload": wl.name, "padded_params": P,
           "kernel_sources_sha256_16": kernel_source_hash(a.record_tag), "launches": n,
           "dram_bytes_read_per_launch": sum(d["dram__bytes_read.sum"] for d in got) / n,
           "dram_bytes_write_per_launch": sum(d["dram__bytes_write.sum"] for d in got) / n,
           "gpu_time_ms_per_launch": sum(d.get("gpu__time_duration.sum", 0.0) for d in got) / n * 1e3,
           "capture": a.record_note}
    out = traffic_record_name(a.record_tag, wl.name)
    with open(out, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    print(json.dumps(rec))


class NvmlClockSampler:
    """SM clock and clock-event-reason samples read through NVML (read-only queries) by a
    polling thread, about every `period` seconds; only those taken between mark_start()
    and mark_end() (the timed region) are summarised.  `nvml` is the pynvml module (a
    stand-in in tests); `index` the NVML index of the GPU."""
    REASON_BITS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
                   ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
                   ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"),
                   ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
                   ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, nvml, index, period=0.002):
        import threading
        self.nvml, self.period = nvml, period
        nvml.nvmlInit()
        self.h = nvml.nvmlDeviceGetHandleByIndex(index)
        self.max_mhz = float(nvml.nvmlDeviceGetMaxClockInfo(self.h, nvml.NVML_CLOCK_SM))
        self.t0 = self.t1 = None
        self.samples = []
        self._sample()                 # a query that fails, fails here (the caller falls back)
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._poll, daemon=True)
        self._thread.start()

    def _sample(self):
        nv = self.nvml
        t = time.time()
        self.samples.append((t, float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)),
                             int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))))

    def _poll(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            self._stop.wait(self.period)

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        self._stop.set()
        self._thread.join(timeout=5)
        try:
            self.nvml.nvmlShutdown()
        except Exception:
            pass
        inside = [x for x in self.samples if self.t0 is not None and self.t0 <= x[0] <= (self.t1 or 1e18)]
        rows = inside or self.samples
        if not rows:
            return None
        bits = {name: getattr(self.nvml, attr) for name, attr in self.REASON_BITS}
        reasons = sorted({name for _, _, r in rows for name, bit in bits.items() if r & bit})
        return {"sm_mhz": statistics.median(sm for _, sm, _ in rows), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(rows), "in_timed_region": bool(inside), "source": "nvml"}


def clock_sampler(cuda_index):
    """NVML polling when the pynvml module and the driver's NVML answer; nvidia-smi
    otherwise."""
    try:
        import pynvml
        import torch
        index = torch.cuda._get_nvml_device_index(cuda_index)
        return NvmlClockSampler(pynvml, index)
    except Exception:
        return ClockSampler(cuda_index)


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples; only those taken between mark_start()
    and mark_end() (the timed region) are summarised."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index):
        self.gpu = str(gpu_index)
        self.t0 = self.t1 = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                       "-lms", "10"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    @staticmethod
    def _when(stamp):
        from datetime import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.strptime(stamp, fmt).timestamp()
            except ValueError:
                pass
        return None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        rows = [[c.strip() for c in r.split(",")] for r in open(self.f.name).read().splitlines() if r.strip()]
        os.unlink(self.f.name)
        rows = [r for r in rows if len(r) >= 10 and r[1] == self.gpu]
        inside = [r for r in rows if self.t0 is not None and self._when(r[0]) is not None
                  and self.t0 - 0.05 <= self._when(r[0]) <= (self.t1 or 1e18) + 0.05]
        rows = inside or rows
        if not rows:
            return None
        num = lambda x: float(x) if x.replace(".", "", 1).isdigit() else None
        sm = [num(r[2]) for r in rows if num(r[2]) is not None]
        reasons = sorted({self.REASONS[j] for r in rows for j in range(4) if r[6 + j].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(rows[0][3]),
                "reasons": reasons, "samples": len(rows), "in_timed_region": bool(inside), "source": "nvidia-smi"}


def workload_config(wl, world):
    return {"workload": wl.name, "description": wl.description, "psi": wl.psi, "n_ranks_simulated": wl.n_ranks,
            "zero_stage": wl.stage, "bucket_elems": wl.bucket_elems, "loss_scale": wl.loss_scale,
            "inputs": "seeded synthetic (Philox4x32-10), resident in HBM",
            "l2": "working set far above the 126 MB L2; no flush needed",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU (ranks simulated in HBM)"}


def variant_config(a, wl, world):
    c = workload_config(wl, world)
    if a.wire_fp16:
        c["ring_partials"] = "fp16 wire"
    if a.dynamic:
        c["step"] = "zero_step_dynamic"
    if a.dynamic_commit:
        c["step"] = "zero_step_dynamic_commit"
    if first_cap(a):
        c["max_ctas"] = first_cap(a)
    return c


def first_cap(a):
    return int(str(a.max_ctas).split(",")[0])


# ---------------------------------------------------------------- CPU oracle sample

def oracle_sample_run(wl, psi_s, steps=1):
    """Run the oracle on the first psi_s parameters of the workload (same N, stage, input
    distributions, hyper-parameters); returns seconds spent in the oracle."""
    import oracle
    import seeded_inputs as si
    from oracle.layout import make_layout
    B = wl.bucket_elems if wl.bucket_elems > 0 else 0
    lay = make_layout([psi_s], wl.n_ranks, B, wl.pad_align)
    P = lay.padded
    g = si.fill_grads(wl.n_ranks, P, psi_s, wl.seed, wl.grad_sigma, wl.loss_scale, wl.heavy_frac, wl.heavy_mult)
    master = si.fill_f32(P, psi_s, wl.seed, si.STREAM_MASTER, wl.master_sigma)
    m = si.fill_f32(P, psi_s, wl.seed, si.STREAM_M, wl.m_sigma) if wl.m_sigma else np.zeros(P, np.float32)
    v = si.fill_f32(P, psi_s, wl.seed, si.STREAM_V, wl.v_sigma, True) if wl.v_sigma else np.zeros(P, np.float32)
    hp = oracle.Hyper(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale)
    t0 = time.perf_counter()
    oracle.run_steps(lay, wl.stage, g, master, m, v, hp, steps)
    return time.perf_counter() - t0


class one_core:
    """Run the oracle pinned to one CPU of this process's allowed set (restored after)."""

    def __enter__(self):
        self.saved = None
        if hasattr(os, "sched_getaffinity"):
            self.saved = os.sched_getaffinity(0)
            os.sched_setaffinity(0, {min(self.saved)})
        return self

    def __exit__(self, *exc):
        if self.saved is not None:
            os.sched_setaffinity(0, self.saved)


def host_info():
    model = ""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model, "pinned_to_one_core": hasattr(os, "sched_setaffinity")}


def size_sample(wl, seconds):
    """Largest power-of-two sample whose one-step oracle run fits `seconds`."""
    psi_s = 1 << 16
    t = oracle_sample_run(wl, psi_s)
    while t * 2 < seconds and psi_s < (1 << 27):
        psi_s *= 2
        t = t * 2
    return psi_s


def cpu_baseline(wl, seconds):
    with one_core():
        psi_s = size_sample(wl, seconds)
        t = oracle_sample_run(wl, psi_s)
    return {"value": psi_s / t, "unit": UNIT, "cores": 1, "kind": "oracle", "host": host_info(),
            "sample": f"first {psi_s} parameters of {wl.name} (same N={wl.n_ranks}, stage {wl.stage}, "
                      f"inputs, AdamW), one step, single-threaded C oracle, {t:.1f} s"}


def run_reference(a, wl):
    rank, _, world = dist_env()
    if rank != 0:
        return
    per_step = a.ref_seconds / (a.steps + a.warmup)
    with one_core():
        psi_s = size_sample(wl, per_step)
        for _ in range(a.warmup):
            oracle_sample_run(wl, psi_s)
        ts = [oracle_sample_run(wl, psi_s) for _ in range(a.steps)]
    t = sum(ts) / len(ts)
    value = psi_s / t
    sample = (f"each step: first {psi_s} parameters of {wl.name} (same N={wl.n_ranks}, stage {wl.stage}, inputs, "
              f"AdamW), single-threaded C oracle")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": workload_config(wl, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
                         "host": host_info()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ---------------------------------------------------------------- the GPU arm

def run_ours(a, wl):
    """The GPU arm: the headline workload, then (default run) the second roofline target
    in the same process, its buffers allocated only after the first's are freed."""
    import torch
    import torch.distributed as dist
    from seeded_inputs.workloads import full_workloads

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize()

    out = _measure(a, wl, world, rank, barrier, headline=True)
    extra = {}
    for name in also_workloads(a):
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        extra[name] = _measure(a, full_workloads()[name], world, rank, barrier, headline=False)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    if extra:
        out["configs"] = extra
    if world == 1 and a.cpu_seconds > 0:
        out["cpu_baseline"] = cpu_baseline(wl, a.cpu_seconds)
    print(json.dumps(out), flush=True)


def also_workloads(a):
    """Workloads timed after the headline in the same run.  By default the plain run of
    the flat 1.3e9 list adds the Llama-shaped ZeRO-3 list: the two fused-step roofline
    targets, both on the clock of one bench invocation."""
    if a.also == "none":
        return []
    if a.also != "auto":
        return [x for x in a.also.split(",") if x]
    variant = a.wire_fp16 or a.dynamic or a.dynamic_commit or a.shrink > 1 or a.psi or a.kernel or a.ranks
    return ["llama3b_n8_zero3"] if a.workload == DEFAULT_WORKLOAD and not variant else []


def _measure(a, wl, world, rank, barrier, headline):
    """Time K fused steps of one workload (after W warm-up steps) with CUDA events, max
    over ranks; the headline also runs the end-to-end host-buffer leg and the requested
    variant (fp16 wire, dynamic scaling).  Returns the JSON fields (rank 0's view)."""
    import torch
    import seeded_inputs as si
    import zero_sharded_optimizer_ring_b200 as zs

    plain = not headline
    lay = zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units),
                    wire_fp16=a.wire_fp16 and not plain)
    lay.to_device()
    if a.kernel:
        lay.set_impl(a.kernel)
    if first_cap(a):
        lay.set_max_ctas(first_cap(a))
    P, psi, N = lay.padded, lay.psi, wl.n_ranks
    g = torch.empty((N, P), dtype=torch.int16, device="cuda")
    si.fill_grads_cuda(g, psi, wl.seed, wl.grad_sigma, wl.loss_scale, wl.heavy_frac, wl.heavy_mult)
    master = torch.empty(P, dtype=torch.float32, device="cuda")
    si.fill_f32_cuda(master, psi, wl.seed, si.STREAM_MASTER, wl.master_sigma)
    m = torch.zeros(P, dtype=torch.float32, device="cuda")
    v = torch.zeros(P, dtype=torch.float32, device="cuda")
    if wl.m_sigma:
        si.fill_f32_cuda(m, psi, wl.seed, si.STREAM_M, wl.m_sigma)
    if wl.v_sigma:
        si.fill_f32_cuda(v, psi, wl.seed, si.STREAM_V, wl.v_sigma, absval=True)
    p16_full = torch.zeros(P, dtype=torch.int16, device="cuda")
    p16_shard = torch.zeros(P, dtype=torch.int16, device="cuda") if wl.stage == 3 else None
    nonfinite = torch.zeros(max(1, lay.n_buckets), dtype=torch.int32, device="cuda")
    dynamic = a.dynamic and not plain
    dynamic_commit = a.dynamic_commit and not plain

    def hp(t):
        return zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale, t)

    if dynamic:
        # the scale the gradients carry never overflows here, so every step applies; the
        # timed work is the reduce-scatter pass, the overflow check (a host round trip)
        # and the update pass
        reduced = torch.empty(P, dtype=torch.float32, device="cuda")
        scaler = zs.LossScaler(wl.loss_scale, window=1 << 40)

        def one_step(t, events=None):
            if events:
                events["update_begin"].record()
            zs.step_dynamic(lay, g, reduced, master, m, v, p16_shard, p16_full, hp(t), scaler, nonfinite)
            if events:
                events["update_end"].record()
    elif dynamic_commit:
        # two state sets and two fp16 parameter buffers; an applied step swaps them (the
        # scale never overflows here, so every step applies)
        scaler = zs.LossScaler(wl.loss_scale, window=1 << 40)
        sets = [[master, m, v], [torch.empty_like(master), torch.empty_like(m), torch.empty_like(v)]]
        p16_sets = [p16_shard if wl.stage == 3 else p16_full, torch.empty_like(p16_full)]

        def one_step(t, events=None):
            if events:
                events["update_begin"].record()
            applied = zs.step_dynamic_commit(lay, g, sets[0], sets[1], p16_sets[1], p16_full, hp(t), scaler,
                                             nonfinite)
            if events:
                events["update_end"].record()
            if applied:
                sets.reverse()
                p16_sets.reverse()
    else:
        def one_step(t, events=None):
            zs.step(lay, g, master, m, v, p16_shard, p16_full, hp(t), nonfinite=nonfinite, events=events)

    t = 0
    for _ in range(a.warmup):
        t += 1
        one_step(t)
    zs.get_error(lay)

    K = a.steps
    ev = [{k: torch.cuda.Event(enable_timing=True) for k in ("update_begin", "update_end", "gather_begin", "gather_end")}
          for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = clock_sampler(torch.cuda.current_device()) if rank == 0 else None
    time.sleep(0.3)
    barrier()
    if sampler:
        sampler.mark_start()
    start.record()
    for i in range(K):
        t += 1
        one_step(t, ev[i])
    end.record()
    barrier()
    if sampler:
        sampler.mark_end()
    clocks = sampler.stop() if sampler else None
    zs.get_error(lay)
    ms = max_over_ranks(start.elapsed_time(end) / K, world, "cuda")
    upd_ms = max_over_ranks(sum(e["update_begin"].elapsed_time(e["update_end"]) for e in ev) / K, world, "cuda")
    gat_ms = None
    if wl.stage == 3 and not (dynamic or dynamic_commit):      # those modes time one bracket
        gat_ms = max_over_ranks(sum(e["gather_begin"].elapsed_time(e["gather_end"]) for e in ev) / K, world, "cuda")
    # our kernels per step: the fused kernel (reduce + update for --dynamic), the gather
    launches_per_step = (2 if dynamic else 1) + (1 if wl.stage == 3 else 0)

    # end to end through the host-buffer entry point: gradients from pinned host memory
    # in, fp16 parameters to pinned host memory out, every step
    e2e = None
    if headline and a.e2e_steps > 0 and not (dynamic or dynamic_commit):
        del g
        torch.cuda.empty_cache()
        g_host = torch.empty((N, P), dtype=torch.int16).pin_memory()
        ge = torch.empty((N, P), dtype=torch.int16, device="cuda")
        si.fill_grads_cuda(ge, psi, wl.seed, wl.grad_sigma, wl.loss_scale, wl.heavy_frac, wl.heavy_mult)
        g_host.copy_(ge)
        p16_host = torch.empty(P, dtype=torch.int16).pin_memory()
        t += 1
        zs.step_host(lay, g_host, ge, master, m, v, p16_shard, p16_full, p16_host, hp(t))
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record()
        for _ in range(a.e2e_steps):
            t += 1
            zs.step_host(lay, g_host, ge, master, m, v, p16_shard, p16_full, p16_host, hp(t))
        e2.record()
        barrier()
        e2e_ms = max_over_ranks(s2.elapsed_time(e2) / a.e2e_steps, world, "cuda")
        e2e = {"value": throughput(psi, world, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": 2 * N * P, "d2h_bytes_per_step": 2 * P,
               "steps": a.e2e_steps, "path": "zero_step_host (pinned host grads in, fp16 params out)"}
        del g_host, p16_host, ge
    lay.close()
    if rank != 0:
        return None

    impl_name = {0: "bulk-copy pipeline (bulk_step_kernel, automatic choice)", 1: "register streaming (tile_kernel)",
                 2: "bulk-copy pipeline (bulk_step_kernel)"}[a.kernel]
    if a.wire_fp16 and not plain:
        impl_name += ", fp16 wire"
    if dynamic:
        impl_name = "dynamic loss scaling: reduce-scatter + overflow check + update (two passes)"
    if dynamic_commit:
        impl_name = "dynamic loss scaling, two-phase commit: fused pass into a second state set + overflow check"
    peak, peak_kind = hbm_peak()
    fused_bytes = fused_bytes_per_param(wl) * P
    if dynamic:
        fused_bytes = (2 * wl.n_ranks + 4 + 4 + 24 + 2) * P     # reduce pass + update pass
    if (dynamic or dynamic_commit) and wl.stage == 3:
        fused_bytes += 4 * P                                    # the events bracket the gather too
    achieved = fused_bytes / (upd_ms / 1e3) / 1e9
    plain_fused = not (dynamic or dynamic_commit or (a.wire_fp16 and not plain))
    kernel_tag = {0: "bulk_step", 1: "tile_kernel", 2: "bulk_step"}[a.kernel]
    traffic = profiled_traffic(kernel_tag, wl.name, P) if plain_fused else None
    step_bytes = ideal_bytes_per_param(wl) * P
    out = {
        "metric": METRIC, "value": throughput(psi, world, ms), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": variant_config(a, wl, world) if headline else workload_config(wl, world),
        "hbm": {"achieved_gbs_step": step_bytes / (ms / 1e3) / 1e9, "ideal_bytes_per_param": ideal_bytes_per_param(wl),
                "frac_of_measured_peak": step_bytes / (ms / 1e3) / 1e9 / peak,
                "frac_of_nominal_8tbs": step_bytes / (ms / 1e3) / 1e9 / NOMINAL_HBM_GBS},
        "roofline": {"bound": "hbm", "kernel": "fused reduce-scatter + AdamW, " + impl_name,
                     "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak, "kernel_ms": upd_ms,
                     "algorithmic_bytes_per_launch": fused_bytes,
                     "traffic": traffic},
        "gpu_launches": K * launches_per_step,
        "clocks": clocks,
    }
    if headline:
        out["e2e"] = e2e
    if gat_ms is not None:
        gather_bytes = 4 * P
        out["gather_kernel_ms"] = gat_ms
        out["gather_gbs"] = gather_bytes / (gat_ms / 1e3) / 1e9
        out["gather_roofline"] = {
            "bound": "hbm", "kernel": "all-gather copy (copy_range_kernel)",
            "achieved": gather_bytes / (gat_ms / 1e3) / 1e9, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
            "frac": gather_bytes / (gat_ms / 1e3) / 1e9 / peak, "kernel_ms": gat_ms,
            "algorithmic_bytes_per_launch": gather_bytes,
            "traffic": profiled_traffic("copy_range", wl.name, P) if plain_fused else None}
    return out


def run_overlap(a, wl):
    """The step overlapped with a simulated backward pass.  The backward writes every
    rank's gradients one bucket at a time, tail bucket first (seeded generator kernels:
    ALU-heavy, like a backward pass, and writing the 2N bytes per parameter a backward
    pass writes), on its own stream, recording an event per bucket; zero_step_overlapped
    runs each bucket's fused update on the compute stream as soon as its event fires."""
    import torch
    import seeded_inputs as si
    import zero_sharded_optimizer_ring_b200 as zs

    torch.cuda.set_device(dist_env()[1])
    lay = zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units))
    lay.to_device()
    if a.kernel:
        lay.set_impl(a.kernel)
    P, psi, N = lay.padded, lay.psi, wl.n_ranks
    g = torch.zeros((N, P), dtype=torch.int16, device="cuda")
    master = torch.empty(P, dtype=torch.float32, device="cuda")
    si.fill_f32_cuda(master, psi, wl.seed, si.STREAM_MASTER, wl.master_sigma)
    m = torch.zeros(P, dtype=torch.float32, device="cuda")
    v = torch.zeros(P, dtype=torch.float32, device="cuda")
    p16_full = torch.zeros(P, dtype=torch.int16, device="cuda")
    p16_shard = torch.zeros(P, dtype=torch.int16, device="cuda") if wl.stage == 3 else None
    _, buckets, _, _ = lay.tables()
    ev = lambda: torch.cuda.Event(enable_timing=True)
    hi_pri = torch.cuda.Stream.priority_range()[1]       # numerically lowest = highest priority
    caps = [int(x) for x in str(a.max_ctas).split(",")]

    def generator_backward(producer):
        def backward(events=None):
            for b, (lo, hi) in enumerate(buckets):
                si.fill_grads_range_cuda(g, int(lo), int(hi), psi, wl.seed, wl.grad_sigma, wl.loss_scale,
                                         wl.heavy_frac, wl.heavy_mult, cuda_stream=producer.cuda_stream)
                if events is not None:
                    events[b].record(producer)
        return backward

    def gemm_backward(producer):
        # per bucket of n_b parameters, viewed as a [D, n_b / D] weight: the activation
        # gradient [T, D] x [D, n] and the weight gradient [D, T] x [T, n], 4 T n_b FLOPs;
        # the gradients themselves are generated once, here, and stay
        si.fill_grads_cuda(g, psi, wl.seed, wl.grad_sigma, wl.loss_scale, wl.heavy_frac, wl.heavy_mult)
        T, D = a.bwd_tokens, 4096
        A = torch.randn(T, D, device="cuda", dtype=torch.bfloat16)
        shapes = [max(128, (int(hi - lo) // D + 127) // 128 * 128) for lo, hi in buckets]
        mats = {n: (torch.randn(D, n, device="cuda", dtype=torch.bfloat16),
                    torch.empty(T, n, device="cuda", dtype=torch.bfloat16),
                    torch.empty(D, n, device="cuda", dtype=torch.bfloat16)) for n in set(shapes)}

        def backward(events=None):
            with torch.cuda.stream(producer):
                for b, n in enumerate(shapes):
                    w, act, wgrad = mats[n]
                    torch.mm(A, w, out=act)
                    torch.mm(A.t(), act, out=wgrad)
                    if events is not None:
                        events[b].record(producer)
        backward.tflop = sum(4.0 * T * D * n for n in shapes) / 1e12
        return backward

    t = 0
    reps = max(3, a.steps // 20)
    groups = [None if x == "auto" else int(x) for x in str(a.bucket_group).split(",")]
    if a.backward == "gemm":
        runs = [("default", 0, cap, grp) for cap in caps for grp in groups]
    else:
        runs = [("default", 0, caps[0], grp) for grp in groups] + [("high", hi_pri, caps[0], groups[0])]
    for prio_name, prio, cap, grp in runs:
        if cap == 0:       # a fresh layout: the overlapped step's grid tuner starts from scratch
            lay.close()
            lay = zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units))
            lay.to_device()
            if a.kernel:
                lay.set_impl(a.kernel)
        lay.set_max_ctas(cap)
        producer, compute = torch.cuda.Stream(), torch.cuda.Stream(priority=prio)
        make = gemm_backward if a.backward == "gemm" else generator_backward
        t = _overlap_reps(a, wl, lay, g, master, m, v, p16_shard, p16_full, make(producer), producer,
                          compute, ev, reps, t, prio_name, cap, grp)
    zs.get_error(lay)


def _overlap_reps(a, wl, lay, g, master, m, v, p16_shard, p16_full, backward, producer, compute, ev, reps, t,
                  prio_name, cap, group):
    import torch
    import zero_sharded_optimizer_ring_b200 as zs

    def hp():
        return zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale, t)

    res = {"bwd": [], "step": [], "seq": [], "pipe": [], "pipe_all": []}
    # the plan tuner: a warm-up call, then every plan timed twice
    warmup = a.warmup if cap else max(a.warmup, 1 + zs._abi.OVERLAP_PLANS * 2 + 1)
    for rep in range(warmup + reps):
        torch.cuda.synchronize()
        s0, e0 = ev(), ev()
        s0.record(producer)
        backward()
        e0.record(producer)
        torch.cuda.synchronize()
        t += 1
        s1, e1 = ev(), ev()
        s1.record(compute)
        zs.step(lay, g, master, m, v, p16_shard, p16_full, hp(), stream=compute)
        e1.record(compute)
        torch.cuda.synchronize()
        t += 1
        # back to back in one timed region: the whole backward, then the whole step, no
        # idle gap between them (the same power and clock state the pipelined run sees)
        s3, e3, done = ev(), ev(), torch.cuda.Event()
        s3.record(producer)
        backward()
        done.record(producer)
        compute.wait_event(done)
        zs.step(lay, g, master, m, v, p16_shard, p16_full, hp(), stream=compute)
        e3.record(compute)
        torch.cuda.synchronize()
        t += 1
        ready = [torch.cuda.Event() for _ in range(lay.n_buckets)]
        s2, e2 = ev(), ev()
        s2.record(producer)
        backward(ready)
        zs.step_overlapped(lay, ready, g, master, m, v, p16_shard, p16_full, hp(), stream=compute, group=group)
        e2.record(compute)
        torch.cuda.synchronize()
        res["pipe_all"].append(round(s2.elapsed_time(e2), 3))
        if rep >= warmup:
            res["bwd"].append(s0.elapsed_time(e0))
            res["step"].append(s1.elapsed_time(e1))
            res["seq"].append(s3.elapsed_time(e3))
            res["pipe"].append(s2.elapsed_time(e2))
    tb, ts, tq, tp = (statistics.median(res[k]) for k in ("bwd", "step", "seq", "pipe"))
    print(json.dumps({
        "metric": "bucket-pipelined step behind a simulated backward (overlap)", "workload": wl.name,
        "backward": a.backward, "compute_stream_priority": prio_name,
        "kernel": {0: "automatic", 1: "register streaming", 2: "bulk-copy pipeline"}[a.kernel],
        "max_ctas": cap if cap else "auto (measured by the library)",
        "bucket_group": group if group else "auto (zero_step_overlapped: launches of >= 2^24 elements)",
        "t_back_to_back_ms": tq, "t_backward_plus_step_alone_ms": tb + ts,
        "chosen_plan": dict(zip(("plan", "mean_ms_per_plan"), lay.overlap_plan())),
        "pipelined_every_call_ms": res["pipe_all"],
        "buckets": lay.n_buckets,
        "reps": reps, "t_backward_ms": tb, "t_step_ms": ts, "t_pipelined_ms": tp, "exposed_step_ms": tp - tb,
        "overlap_efficiency": (tb + ts - tp) / ts,
        **({"backward_tflops": backward.tflop / (tb / 1e3)} if hasattr(backward, "tflop") else {}),
        "note": "overlap_efficiency = share of the step hidden behind the backward (1 = fully hidden)"}),
        flush=True)
    return t


def run_graph(a, wl):
    """Launch-bound small models: K fused steps launched one by one (zero_step, scalars
    passed at launch) against the same K steps replayed from CUDA graphs, each graph
    holding G captured steps of zero_step_device_scalars that read their scalars from rows
    of a device table filled before timing.  Both timed with CUDA events on one stream,
    inputs resident, the same kernels."""
    import torch
    import seeded_inputs as si
    import zero_sharded_optimizer_ring_b200 as zs

    torch.cuda.set_device(dist_env()[1])
    lay = zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units))
    lay.to_device()
    P, psi, N = lay.padded, lay.psi, wl.n_ranks
    g = torch.empty((N, P), dtype=torch.int16, device="cuda")
    si.fill_grads_cuda(g, psi, wl.seed, wl.grad_sigma, wl.loss_scale, wl.heavy_frac, wl.heavy_mult)
    master = torch.empty(P, dtype=torch.float32, device="cuda")
    si.fill_f32_cuda(master, psi, wl.seed, si.STREAM_MASTER, wl.master_sigma)
    m = torch.zeros(P, dtype=torch.float32, device="cuda")
    v = torch.zeros(P, dtype=torch.float32, device="cuda")
    p16_full = torch.zeros(P, dtype=torch.int16, device="cuda")
    p16_shard = torch.zeros(P, dtype=torch.int16, device="cuda") if wl.stage == 3 else None
    hp = lambda t: zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale, t)
    G = max(1, min(a.graph_steps, a.steps))
    K = (a.steps // G) * G
    st = torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)
    t = 0
    with torch.cuda.stream(st):
        for _ in range(a.warmup):
            t += 1
            zs.step(lay, g, master, m, v, p16_shard, p16_full, hp(t))
        torch.cuda.synchronize()
        s0, e0 = ev(), ev()
        s0.record()
        for _ in range(K):
            t += 1
            zs.step(lay, g, master, m, v, p16_shard, p16_full, hp(t))
        e0.record()
        torch.cuda.synchronize()
    plain_ms = s0.elapsed_time(e0) / K

    # the scalars of the next K steps in a device table; graph i holds steps i*G .. i*G+G-1,
    # each reading its own row (a training loop would refill one table per replay instead)
    table = torch.empty((K, 9), dtype=torch.float32, device="cuda")
    table.copy_(torch.from_numpy(np.stack([zs.step_scalars(lay, hp(t + 1 + k)) for k in range(K)])))
    t += K
    graphs = []
    for i in range(K // G):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=st):
            for j in range(G):
                zs.step_device_scalars(lay, g, master, m, v, p16_shard, p16_full, table[i * G + j])
        graphs.append(gr)
    torch.cuda.synchronize()
    s1, e1 = ev(), ev()
    with torch.cuda.stream(st):
        s1.record()
        for gr in graphs:
            gr.replay()
        e1.record()
        torch.cuda.synchronize()
    graph_ms = s1.elapsed_time(e1) / K
    zs.get_error(lay)
    del graphs
    print(json.dumps({"metric": "fused step launched per step vs replayed from a CUDA graph", "workload": wl.name,
                      "psi": psi, "steps": K, "steps_per_graph": G, "plain_ms_per_step": plain_ms,
                      "graph_ms_per_step": graph_ms, "plain_params_per_s": psi / (plain_ms / 1e3),
                      "graph_params_per_s": psi / (graph_ms / 1e3),
                      "note": "scalars of every step in a device table filled before timing"}), flush=True)


def run_unfused(a, wl):
    """The three standalone boundary calls of one step, each timed with CUDA events:
    zero_reduce_scatter of every bucket (2N + 4 bytes per parameter: fp16 grads in, fp32
    sums out), zero_adamw_shard_step of every shard (4 + 24 + 2: sums, state, fp16
    parameters) and zero_allgather of every unit (2 + 2).  The fused step moves 2N + 26."""
    import torch
    import seeded_inputs as si
    import zero_sharded_optimizer_ring_b200 as zs

    torch.cuda.set_device(dist_env()[1])
    lay = zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units))
    lay.to_device()
    if a.kernel:
        lay.set_impl(a.kernel)
    P, psi, N = lay.padded, lay.psi, wl.n_ranks
    g = torch.empty((N, P), dtype=torch.int16, device="cuda")
    si.fill_grads_cuda(g, psi, wl.seed, wl.grad_sigma, wl.loss_scale, wl.heavy_frac, wl.heavy_mult)
    master = torch.empty(P, dtype=torch.float32, device="cuda")
    si.fill_f32_cuda(master, psi, wl.seed, si.STREAM_MASTER, wl.master_sigma)
    m = torch.zeros(P, dtype=torch.float32, device="cuda")
    v = torch.zeros(P, dtype=torch.float32, device="cuda")
    if wl.m_sigma:
        si.fill_f32_cuda(m, psi, wl.seed, si.STREAM_M, wl.m_sigma)
    if wl.v_sigma:
        si.fill_f32_cuda(v, psi, wl.seed, si.STREAM_V, wl.v_sigma, absval=True)
    red = torch.empty(P, dtype=torch.float32, device="cuda")
    p16 = torch.zeros(P, dtype=torch.int16, device="cuda")
    p16_full = torch.zeros(P, dtype=torch.int16, device="cuda")
    hp = lambda t: zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale, t)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    times = {"reduce_scatter": [], "adamw": [], "allgather": []}
    for t in range(1, a.warmup + a.steps + 1):
        e = [ev() for _ in range(4)]
        e[0].record()
        zs.reduce_scatter(lay, -1, g, red)
        e[1].record()
        zs.adamw_shard_step(lay, -1, red, master, m, v, p16, hp(t))
        e[2].record()
        zs.allgather(lay, -1, p16, p16_full)
        e[3].record()
        if t > a.warmup:
            torch.cuda.synchronize()
            for k, (i, j) in zip(times, ((0, 1), (1, 2), (2, 3))):
                times[k].append(e[i].elapsed_time(e[j]))
    zs.get_error(lay)
    peak, peak_kind = hbm_peak()
    out = {"metric": "standalone boundary calls of one step", "workload": wl.name, "steps": a.steps,
           "peak": peak, "peak_kind": peak_kind}
    for k, per_param in (("reduce_scatter", 2 * N + 4), ("adamw", 4 + 24 + 2), ("allgather", 4)):
        ms = statistics.median(times[k])
        gbs = per_param * P / (ms / 1e3) / 1e9
        out[k] = {"ms": ms, "bytes_per_param": per_param, "achieved_gbs": gbs, "frac": gbs / peak}
    out["unfused_step_ms"] = sum(out[k]["ms"] for k in times)
    print(json.dumps(out), flush=True)


def run_zero3_passes(a, wl):
    """ZeRO-3's gather passes over the Llama-shaped list: each layer's parameters are
    gathered (zero_gather_unit) into one of n_slots unit-sized buffers and the layer's
    matrices are then used by a simulated compute: one GEMM per matrix with T tokens in the
    forward pass, two (input and weight gradients) in the backward pass (cuBLAS, standing
    in for the model).  Reported: each pass with 1, 2 and 3 slots (1 = no prefetch), the
    compute alone (parameters already in place) and the gathers alone."""
    import torch
    import zero_sharded_optimizer_ring_b200 as zs
    from zero_sharded_optimizer_ring_b200.schedule import GatherWidth, layer_breakdown, zero3_pass
    from seeded_inputs.workloads import llama_tensors

    torch.cuda.set_device(dist_env()[1])
    d, ffn, vocab, layers = 3072, 8192, 32000, 26
    tensors, units = llama_tensors(vocab, d, ffn, layers)
    if tuple(tensors) != tuple(wl.tensors):
        raise SystemExit("--zero3-passes needs the Llama-shaped workload")
    lay = zs.Layout(list(tensors), wl.n_ranks, 3, wl.bucket_elems, wl.pad_align, list(units)).to_device()
    P = lay.padded
    shard = (torch.randn(P, device="cuda", dtype=torch.float16) * 0.02).view(torch.int16)
    _, _, _, u = lay.tables()
    width = int(max(hi - lo for lo, hi in u))
    # matrices of a layer unit: (offset in the unit, rows, cols); norms carry no GEMM
    layer_mats, off = [], d
    for rows, cols in [(d, d)] * 4:
        layer_mats.append((off, rows, cols))
        off += rows * cols
    off += d
    for rows, cols in [(ffn, d), (ffn, d), (d, ffn)]:
        layer_mats.append((off, rows, cols))
        off += rows * cols
    T = a.tokens
    x = {d: torch.randn(T, d, device="cuda", dtype=torch.float16),
         ffn: torch.randn(T, ffn, device="cuda", dtype=torch.float16)}
    gy = {d: torch.randn(T, d, device="cuda", dtype=torch.float16),
          ffn: torch.randn(T, ffn, device="cuda", dtype=torch.float16)}

    def mats(unit, buf):
        if unit == 0 or unit == lay.n_units - 1:
            return []                                  # embedding lookup / final norm: no GEMM
        w = buf.view(torch.float16)
        return [w[o:o + r * c].view(r, c) for o, r, c in layer_mats]

    def fwd(unit, buf):
        for W in mats(unit, buf):
            torch.matmul(x[W.shape[1]], W.t())

    def bwd(unit, buf):
        for W in mats(unit, buf):
            torch.matmul(gy[W.shape[0]], W)            # input gradient
            torch.matmul(gy[W.shape[0]].t(), x[W.shape[1]])   # weight gradient

    ev = lambda: torch.cuda.Event(enable_timing=True)
    gs, cs = torch.cuda.Stream(), torch.cuda.Stream()
    slots = [torch.empty(width, dtype=torch.int16, device="cuda") for _ in range(3)]
    full = torch.empty(P, dtype=torch.int16, device="cuda")
    zs.allgather(lay, -1, shard, full)
    torch.cuda.synchronize()
    order_f = list(range(lay.n_units))
    order_b = order_f[::-1]

    def timed(fn, breakdown=False):
        """Best of 3 repetitions after the warm-up; with breakdown, fn returns the pass's
        events and the per-layer breakdown of the best repetition comes back too."""
        best, best_bd = None, None
        for rep in range(a.warmup + 3):
            torch.cuda.synchronize()
            s0, e0 = ev(), ev()
            s0.record(gs)
            cs.wait_event(s0)
            marks = fn()
            e0.record(cs)
            torch.cuda.synchronize()
            if rep >= a.warmup:
                t = s0.elapsed_time(e0)
                if best is None or t < best:
                    best = t
                    best_bd = layer_breakdown(marks, s0) if breakdown else None
        return (best, best_bd) if breakdown else best

    def compute_only(work):
        def run():
            with torch.cuda.stream(cs):
                for k in order_f:
                    lo, hi = int(u[k][0]), int(u[k][1])
                    work(k, full[lo:hi])
        return run

    def gathers_only():
        for k in order_f:
            zs.gather_unit(lay, k, shard, slots[k % 3], stream=gs)
        cs.wait_stream(gs)

    def short(bd):
        return {k: round(v, 4) for k, v in bd.items() if k.startswith("sum_")} | {
            "max_wait_ms": round(max(bd["wait_ms"]), 4),
            "layers_waiting": sum(1 for w in bd["wait_ms"] if w > 0.005),
            "wait_ms_per_unit": [round(w, 3) for w in bd["wait_ms"]]}

    set_carveout = torch._C._set_sm_carveout_experimental
    passes = (("forward", fwd, order_f), ("backward", bwd, order_b))
    res = {"gathers_only_ms": timed(gathers_only)}
    for gcap in (8, 16, 32):                       # the 28 gathers alone on a capped grid
        lay.set_gather_ctas(gcap)
        res[f"gathers_only_{gcap}ctas_ms"] = timed(gathers_only)
        res[f"gathers_only_{gcap}ctas_gbs"] = 4 * P / (res[f"gathers_only_{gcap}ctas_ms"] / 1e3) / 1e9
    lay.set_gather_ctas(0)
    for name, work, order in passes:
        res[f"{name}_compute_only_ms"] = timed(compute_only(work))
        for n in (1, 2, 3):
            t, bd = timed(lambda: zero3_pass(lay, shard, slots[:n], order, work, gs, cs, gather_ctas=0,
                                             matmul_sm_carveout=None, blas=None), breakdown=True)
            res[f"{name}_{n}slot_ms"] = t
            res[f"{name}_{n}slot_breakdown"] = short(bd)
        for n in (1, 2):
            res[f"{name}_exposed_gather_{n}slot_ms"] = res[f"{name}_{n}slot_ms"] - res[f"{name}_compute_only_ms"]

    # gathers on a capped grid beside GEMMs run with a lowered SM-count target: configurations
    # "carveout:gather_ctas:slots" (carveout = how far below the SM count the matmuls'
    # cuBLAS SM-count target is set; gather_ctas = zero_set_gather_ctas; slots 0 = compute
    # alone), each
    # measured once per round, rounds interleaved so that clock drift hits all alike;
    # reported: the median over rounds
    sweep = []
    # "default" = zero3_pass with its own defaults (capped gathers, matmul SM carveout,
    # cuBLASLt), two slots
    # "width" = the same with the capped gathers' grid chosen per pass kind by feedback
    # (schedule.GatherWidth, kept across rounds after warm-up passes)
    configs = [(c, c, 2) if c in ("default", "width") else tuple(int(x) for x in c.split(":"))
               for c in a.zero3_configs.split(",") if c]
    widths = {name: GatherWidth() for name, _, _ in passes}
    if configs:
        if a.blas:
            torch.backends.cuda.preferred_blas_library(a.blas)
        if any(c == "width" for c, _, _ in configs):
            for _ in range(len(widths["forward"].candidates) * widths["forward"].trials + 2):
                for name, work, order in passes:
                    zero3_pass(lay, shard, slots[:2], order, work, gs, cs, gather_ctas=widths[name])
                    torch.cuda.synchronize()
        rounds = {}
        for rnd in range(a.zero3_rounds):
            for c, gcap, n in configs:
                dflt = c in ("default", "width")
                set_carveout(None if dflt or c == 0 else c)
                lay.set_gather_ctas(0 if dflt else gcap)
                for name, work, order in passes:
                    if n == 0:
                        fn = compute_only(work)
                    elif c == "width":
                        fn = (lambda o=order, w=work, k=n, gw=widths[name]: zero3_pass(lay, shard, slots[:k], o, w, gs,
                                                                                       cs, gather_ctas=gw))
                    elif dflt:
                        fn = (lambda o=order, w=work, k=n: zero3_pass(lay, shard, slots[:k], o, w, gs, cs))
                    else:
                        fn = (lambda o=order, w=work, k=n, gc=gcap: zero3_pass(lay, shard, slots[:k], o, w, gs, cs,
                                                                               gather_ctas=gc, matmul_sm_carveout=None,
                                                                               blas=None))
                    torch.cuda.synchronize()
                    s0, e0 = ev(), ev()
                    s0.record(gs)
                    cs.wait_event(s0)
                    marks = fn()
                    e0.record(cs)
                    torch.cuda.synchronize()
                    bd = layer_breakdown(marks, s0) if n else None
                    rounds.setdefault((c, gcap, n, name), []).append((s0.elapsed_time(e0), bd))
        set_carveout(None)
        lay.set_gather_ctas(0)
        for c, gcap, n in configs:
            row = {"carveout_sms": c, "gather_ctas": gcap, "slots": n}
            for name, _, _ in passes:
                runs = sorted(rounds[(c, gcap, n, name)], key=lambda x: x[0])
                t_med, bd = runs[len(runs) // 2]
                row[f"{name}_ms"] = round(t_med, 4)
                if bd:
                    row[f"{name}_breakdown"] = short(bd)
            sweep.append(row)
        base = {name: statistics.median(t for t, _ in rounds[(0, 0, 0, name)]) for name, _, _ in passes
                } if (0, 0, 0) in configs else None
        if base:
            for row in sweep:
                for name in base:
                    row[f"{name}_exposed_ms"] = round(row[f"{name}_ms"] - base[name], 4)
    gather_bytes = 4 * P
    print(json.dumps({"metric": "ZeRO-3 per-layer gather passes with prefetch", "workload": wl.name,
                      "units": lay.n_units, "tokens": T, "gather_bytes_per_pass": gather_bytes,
                      "gather_gbs": gather_bytes / (res["gathers_only_ms"] / 1e3) / 1e9,
                      **{k: (round(v, 4) if isinstance(v, float) else v) for k, v in res.items()},
                      "sweep": sweep,
                      "gather_width": {name: {"chosen_ctas": w.ctas if w.chosen is not None else None,
                                              "mean_pass_ms": dict(zip(w.candidates, w.means()))}
                                       for name, w in widths.items() if any(w.count)}}), flush=True)


def main():
    a = parse()
    from seeded_inputs.workloads import full_workloads
    wl = full_workloads()[a.workload]
    if a.shrink > 1:
        wl = wl.with_(tensors=tuple(max(1, t // a.shrink) for t in wl.tensors), name=f"{wl.name}_shrink{a.shrink}")
    if a.ranks:
        wl = wl.with_(n_ranks=a.ranks, name=f"{wl.name}_ranks{a.ranks}")
    if a.psi:
        if len(wl.tensors) != 1:
            raise SystemExit("--psi applies to flat (single-tensor) workloads only")
        wl = wl.with_(tensors=(a.psi,), name=f"{wl.name}_psi{a.psi}")
    if a.record_traffic:
        record_traffic(a, wl)
    elif a.impl == "reference":
        run_reference(a, wl)
    elif a.overlap:
        run_overlap(a, wl)
    elif a.graph:
        run_graph(a, wl)
    elif a.unfused:
        run_unfused(a, wl)
    elif a.zero3_passes:
        run_zero3_passes(a, wl)
    else:
        run_ours(a, wl)


if __name__ == "__main__":
    main()
