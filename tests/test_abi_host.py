"""CPU checks of the C ABI: the library loads and exports every function include/zero.h
declares; its host partitioner and counters equal the oracle's; bad arguments are
rejected before anything runs.  No kernel is launched here."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from oracle.layout import make_layout
from seeded_inputs.workloads import full_workloads, reduced_workloads
import zero_sharded_optimizer_ring_b200 as zs
from zero_sharded_optimizer_ring_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build_all()


def _declared():
    src = open(os.path.join(ROOT, "include", "zero.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(zero_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_function():
    names = _declared()
    assert len(names) >= 15
    for path in (build.LIB, build.LIB_DEBUG):      # the release library and its bounds-checking twin
        lib = ctypes.CDLL(path)
        for n in names:
            assert hasattr(lib, n), (path, n)
    assert set(names) == set(_abi.SIGNATURES)


def test_status_codes_named_in_the_binding_and_the_library():
    src = open(os.path.join(ROOT, "include", "zero.h")).read()
    codes = {int(v): k for k, v in re.findall(r"\b(ZERO_(?:OK|ERR_[A-Z]+))\s*=\s*(\d+)", src)}
    assert codes == _abi.STATUS_NAMES
    lib = _abi.lib()
    for c in codes:
        assert lib.zero_status_string(c).decode() != "unknown status", codes[c]


def test_header_constants_mirrored_in_the_binding():
    """Sizes the binding allocates for the library (the plan-mean array of
    zero_overlap_plan) and limits it checks must equal the header's."""
    src = open(os.path.join(ROOT, "include", "zero.h")).read()
    consts = {k: int(v) for k, v in re.findall(r"#define (ZERO_[A-Z_]+) (\d+)", src)}
    assert consts["ZERO_OVERLAP_PLANS"] == _abi.OVERLAP_PLANS
    assert consts["ZERO_NOALLOC_MAX_SEGMENTS"] == _abi.NOALLOC_MAX_SEGMENTS


def test_overlap_plan_before_any_overlapped_call():
    """No plan chosen yet (-1) and every mean 0, in an array of ZERO_OVERLAP_PLANS."""
    lay = zs.Layout([1000], 2, 1, 0, 128, [0])
    plan, means = lay.overlap_plan()
    assert plan == -1 and means == [0.0] * _abi.OVERLAP_PLANS
    lay.close()


def _compare(tensors, N, stage, B, A, units):
    ref = make_layout(tensors, N, B, A, units)
    lay = zs.Layout(tensors, N, stage, B, A, units)
    assert (lay.psi, lay.shard, lay.padded) == (ref.psi, ref.shard, ref.padded)
    t, b, s, u = lay.tables()
    assert list(t) == ref.tensor_off
    assert [tuple(x) for x in b] == ref.buckets
    assert [tuple(x) for x in s] == [tuple(x) for x in ref.segments]
    assert [tuple(x) for x in u] == ref.units
    c = lay.counters()
    rc = oracle.counters(ref, stage)
    assert (c["mem_p16"], c["mem_g16"], c["mem_os"], c["mem_total"], c["sent_elems"], c["recv_elems"]) == \
        (rc.mem_p16, rc.mem_g16, rc.mem_os, rc.mem_total, rc.sent_elems, rc.recv_elems)
    # tile numbering: each segment's tiles are the kTileElems cells it overlaps
    T = lay.tile_elems
    assert lay.n_tiles == sum(-(-hi // T) - lo // T for _, _, lo, hi in ref.segments)
    lay.close()


def test_layout_matches_oracle_random():
    rng = np.random.default_rng(21)
    for _ in range(300):
        N = int(rng.integers(1, 20))
        nt = int(rng.integers(0, 8))
        tensors = [int(x) for x in rng.integers(0, 5000, nt)]
        units = sorted({0} | {int(x) for x in rng.integers(0, max(1, nt), 3)}) if nt and rng.random() < 0.5 else []
        _compare(tensors, N, int(rng.integers(0, 4)), int(rng.integers(-5, 9000)),
                 int(rng.choice([1, 3, 8, 128])), units)


def test_layout_matches_oracle_workloads():
    for wl in list(reduced_workloads().values()) + list(full_workloads().values()):
        _compare(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units))


def test_config_sizes():
    # shard and padding of the flat 1.3e9 workload and the Llama-shaped list
    w = full_workloads()
    lay = zs.Layout(w["flat1p3b_n4_zero1"].tensors, 4, 1, 50_000_000)
    assert (lay.shard, lay.padded, lay.n_buckets) == (325_000_064, 1_300_000_256, 27)
    ll = w["llama3b_n8_zero3"]
    lay = zs.Layout(ll.tensors, 8, 3, 50_000_000, 128, ll.units)
    assert (lay.psi, lay.padded, lay.n_units) == (3_042_868_224, 3_042_868_224, 28)


@pytest.mark.parametrize("kw", [
    dict(n_ranks=0), dict(stage=4), dict(stage=-1), dict(pad_align=0),
    dict(tensors=[5, -1]), dict(units=[1]), dict(units=[0, 0]), dict(units=[0, 9]),
])
def test_invalid_descriptions_rejected(kw):
    args = dict(tensors=[100, 50], n_ranks=2, stage=1, bucket_elems=10, pad_align=8, units=())
    args.update(kw)
    with pytest.raises(zs.ZeroError) as e:
        zs.Layout(**args)
    assert e.value.status == 1


def test_device_calls_need_upload():
    lay = zs.Layout([1000], 2, 1, 100)
    with pytest.raises(zs.ZeroError) as e:
        zs.reduce_scatter(lay, -1, 0, 0, rank_stride=1024, stream=0)
    assert e.value.status == 6           # ZERO_ERR_STATE, nothing launched


def test_empty_layout():
    lay = zs.Layout([], 4, 2, 100)
    assert (lay.psi, lay.padded, lay.n_buckets, lay.n_segments, lay.n_units, lay.n_tiles) == (0, 0, 0, 0, 0, 0)
    lay = zs.Layout([0, 0], 3, 3, 0)
    assert lay.padded == 0


def test_tuning_setters_validate_arguments():
    lay = zs.Layout([1000], 2, 1, 100)
    lay.set_max_ctas(0)
    lay.set_max_ctas(37)
    lay.set_impl(2)
    lay.set_gather_ctas(0)
    lay.set_gather_ctas(16)
    for bad in (lambda: lay.set_max_ctas(-1), lambda: lay.set_impl(3), lambda: lay.set_impl(-1),
                lambda: lay.set_gather_ctas(-1)):
        with pytest.raises(zs.ZeroError) as e:
            bad()
        assert e.value.status == 1


DEVICE_CALLS = ["zero_reduce_scatter", "zero_adamw_shard_step", "zero_allgather", "zero_gather_unit",
                "zero_gather_unit_ranks", "zero_step", "zero_step_bucket", "zero_step_overlapped",
                "zero_step_overlapped_grouped", "zero_step_dynamic", "zero_step_dynamic_commit", "zero_step_host",
                "zero_step_ranks", "zero_step_shard", "zero_step_shard_commit", "zero_copy_shard",
                "zero_layout_device_segments", "zero_get_error", "zero_debug_set_wait"]


@pytest.mark.parametrize("name", DEVICE_CALLS)
def test_device_calls_refuse_a_layout_not_on_the_device(name):
    """Every device entry point checks its layout (and arguments) before any CUDA call:
    with a layout never uploaded it returns INVALID or STATE here, where no GPU exists
    (a CUDA call would have answered ZERO_ERR_CUDA).  zero_step_noalloc is the one entry
    that needs no upload, so it is not in the list."""
    lay = zs.Layout([1000, 24], 2, 1, 100)
    fn = getattr(_abi.lib(), name)
    hp = _abi.AdamWHparams(1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0, 1)
    sc = _abi.LossScaler(1024.0, 2.0, 10, 1.0, 0, 0, 0)
    args = []
    for t in fn.argtypes:
        if t is _abi.ctypes.POINTER(_abi.AdamWHparams):
            args.append(ctypes.byref(hp))
        elif t is _abi.ctypes.POINTER(_abi.LossScaler):
            args.append(ctypes.byref(sc))
        elif t in (ctypes.c_int32, ctypes.c_int64):
            args.append(0)
        elif t is ctypes.c_void_p:
            args.append(None)
        else:
            args.append(t())                                # a NULL pointer of that type
    args[0] = lay.handle
    assert fn(*args) in (1, 6), name                       # ZERO_ERR_INVALID or ZERO_ERR_STATE
    assert (sc.step, sc.skipped) == (0, 0)


def test_scaler_advance_follows_the_oracle_scaler():
    """zero_loss_scaler_advance (the library's scaler rules, also used inside the dynamic
    steps) against the oracle's LossScaler, over a long random skip / apply sequence that
    reaches the floor and several growths; invalid arguments are refused."""
    rng = np.random.default_rng(5)
    lib_sc = zs.LossScaler(2.0 ** 10, factor=2.0, window=4, min_scale=0.5)
    ref = oracle.LossScaler(2.0 ** 10, factor=2.0, window=4, min_scale=0.5)
    seen_floor = grew = 0
    for i in range(2000):
        overflow = bool(rng.random() < (0.6 if i < 300 else 0.1))
        before = ref.scale
        lib_sc.advance(not overflow)
        ref.update(overflow)
        seen_floor += ref.scale == 0.5
        grew += ref.scale > before
        assert (lib_sc.scale, lib_sc.clean_steps, lib_sc.step, lib_sc.skipped) == \
            (ref.scale, ref.clean_steps, ref.step, ref.skipped), i
    assert seen_floor and grew > 5
    with pytest.raises(zs.ZeroError):
        zs.LossScaler(0.0).advance(True)                    # scale must be > 0
    with pytest.raises(zs.ZeroError):
        zs.LossScaler(8.0, factor=1.0).advance(False)       # factor must be > 1


def test_step_scalars_fill_equals_the_oracle_scalars():
    """zero_step_scalars_fill (the library's host computation of a step's nine fp32
    scalars, the values zero_step_device_scalars reads) against the oracle's, bit for bit."""
    for wl in reduced_workloads().values():
        lay = zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units))
        for t in (1, 2, 7, 1000):
            got = zs.step_scalars(lay, zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale, t))
            want = oracle.adamw_scalars(wl.n_ranks, oracle.Hyper(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay,
                                                                   wl.loss_scale), t)
            assert got.view(np.uint32).tolist() == want.view(np.uint32).tolist(), (wl.name, t)
