"""GPU parity: the CUDA path, through the C ABI, against the CPU oracle.

- reduced-size twins of every workload: every element of every output after all steps;
- the full-size workloads in the launch configuration the benchmark times: sampled
  elements (every segment, shard, bucket and unit edge plus random ones) against the
  oracle's per-element path;
- edge cases: one rank, unaligned segment edges (shard rounding 1), one-element
  buckets, a rank count without a compiled specialisation, empty layouts, non-finite
  gradients, zero and -0 operands, capped grids, a flat buffer of more than 2^32
  elements, per-bucket / per-shard / per-unit calls, the host-buffer step.
"""
import numpy as np
import pytest

import oracle
from seeded_inputs.workloads import Workload, full_workloads, reduced_workloads
import zero_sharded_optimizer_ring_b200 as zs
import support as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _hp(wl, t):
    return zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale, t)


def _layout(wl, impl=zs.IMPL_REGISTER):
    lay = zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align,
                    list(wl.units)).to_device()
    lay.set_impl(impl)
    return lay


IMPLS = [zs.IMPL_REGISTER, zs.IMPL_BULK]


def _bufs(lay, wl, rank_stride=None, guard=False):
    """Device inputs and zeroed outputs; with guard=True every written buffer sits between
    guard regions (S.Guarded), checked by _run after each step."""
    g, master, m, v = S.device_inputs(wl, lay.padded, rank_stride)
    p16_shard = torch.zeros(lay.padded, dtype=torch.int16, device="cuda")
    p16_full = torch.zeros(lay.padded, dtype=torch.int16, device="cuda")
    nonfinite = torch.zeros(max(1, lay.n_buckets), dtype=torch.int32, device="cuda")
    b = dict(g=g, master=master, m=m, v=v, p16_shard=p16_shard, p16_full=p16_full, nonfinite=nonfinite)
    b["_guards"] = S.guard_outputs(b) if guard else {}
    return b


def _run(lay, wl, b, steps):
    for t in range(1, steps + 1):
        b["nonfinite"].zero_()
        zs.step(lay, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"], _hp(wl, t),
                nonfinite=b["nonfinite"])
        if b["_guards"]:
            S.assert_guards_intact(b["_guards"], f"step {t}")
    zs.get_error(lay)
    torch.cuda.synchronize()


def _np(t):
    a = t.cpu().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a


def _check_full(wl, lay, b, ref, exact=True):
    S.assert_f32_close(_np(b["master"]), ref.master, "master")
    S.assert_f32_close(_np(b["m"]), ref.m, "m")
    S.assert_f32_close(_np(b["v"]), ref.v, "v")
    S.assert_f16_ulp(_np(b["p16_full"]), ref.p16_full, "p16_full")
    if wl.stage == 3:
        S.assert_f16_ulp(_np(b["p16_shard"]), ref.p16_shard, "p16_shard")
    assert list(_np(b["nonfinite"])[:lay.n_buckets]) == list(ref.nonfinite)
    if exact:
        S.assert_bits_equal(_np(b["master"]), ref.master, "master")
        S.assert_bits_equal(_np(b["m"]), ref.m, "m")
        S.assert_bits_equal(_np(b["v"]), ref.v, "v")
        S.assert_bits_equal(_np(b["p16_full"]), ref.p16_full, "p16_full")


def _oracle(wl, steps=None):
    lay = S.oracle_layout(wl)
    g, master, m, v = S.host_inputs(wl, lay.padded)
    return oracle.run_steps(lay, wl.stage, g, master, m, v, S.hyper(wl), steps or wl.steps), lay


@pytest.fixture(autouse=True)
def _free():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


# ------------------------------------------------------------- reduced-size, every element

@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("key", list(reduced_workloads()))
def test_reduced_workload_all_elements(key, impl):
    wl = reduced_workloads()[key]
    ref, olay = _oracle(wl)
    lay = _layout(wl, impl)
    assert lay.n_tiles >= 8 and lay.n_buckets >= 1     # several tiles, ragged edges
    b = _bufs(lay, wl, guard=True)
    _run(lay, wl, b, wl.steps)
    _check_full(wl, lay, b, ref)

    # ring sums: bit-exact
    red = torch.zeros(lay.padded, dtype=torch.float32, device="cuda")
    nf = torch.zeros(max(1, lay.n_buckets), dtype=torch.int32, device="cuda")
    zs.reduce_scatter(lay, -1, b["g"], red, nonfinite=nf)
    S.assert_bits_equal(_np(red), ref.reduced, "reduced")
    assert list(_np(nf)[:lay.n_buckets]) == list(ref.nonfinite)


@pytest.mark.parametrize("key", list(reduced_workloads()))
def test_unfused_path_matches_oracle(key):
    """The three standalone boundary calls, one bucket / shard / unit at a time:
    zero_reduce_scatter per bucket, zero_adamw_shard_step per shard, zero_allgather per
    unit (stage 3), against the oracle's whole steps, bit for bit."""
    wl = reduced_workloads()[key]
    steps = 2
    ref, _ = _oracle(wl, steps)
    lay = _layout(wl)
    b = _bufs(lay, wl)
    red = torch.zeros(lay.padded, dtype=torch.float32, device="cuda")
    for t in range(1, steps + 1):
        b["nonfinite"].zero_()
        for bk in range(lay.n_buckets):
            zs.reduce_scatter(lay, bk, b["g"], red, nonfinite=b["nonfinite"])
        for k in range(lay.n_ranks):
            out = b["p16_shard"] if wl.stage == 3 else b["p16_full"]
            zs.adamw_shard_step(lay, k, red, b["master"], b["m"], b["v"], out, _hp(wl, t))
        if wl.stage == 3:
            for u in range(lay.n_units):
                zs.allgather(lay, u, b["p16_shard"], b["p16_full"])
    torch.cuda.synchronize()
    S.assert_bits_equal(_np(red), ref.reduced, "reduced (last step)")
    _check_full(wl, lay, b, ref)
    if wl.stage == 3:
        S.assert_bits_equal(_np(b["p16_shard"]), ref.p16_shard, "p16_shard")


def test_deterministic_rerun():
    wl = reduced_workloads()["ragged2000_n16_zero2"]
    lay = _layout(wl)
    outs = []
    for _ in range(2):
        b = _bufs(lay, wl)
        _run(lay, wl, b, 2)
        outs.append({k: _np(v) for k, v in b.items() if k not in ("g", "_guards")})
    for k in outs[0]:
        S.assert_bits_equal(outs[0][k], outs[1][k], k)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("key", ["flat1p3b_n4_zero1", "ragged2000_n16_zero2", "llama3b_n8_zero3"])
def test_capped_grid_matches_oracle(key, impl):
    """zero_set_max_ctas: any grid size deals the same tiles, so every cap gives the
    oracle's result bit for bit (one CTA walks every tile)."""
    wl = reduced_workloads()[key]
    ref, _ = _oracle(wl)
    lay = _layout(wl, impl)
    for cap in (1, 7, 37):
        lay.set_max_ctas(cap)
        b = _bufs(lay, wl)
        _run(lay, wl, b, wl.steps)
        _check_full(wl, lay, b, ref)
        red = torch.zeros(lay.padded, dtype=torch.float32, device="cuda")
        zs.reduce_scatter(lay, -1, b["g"], red)
        S.assert_bits_equal(_np(red), ref.reduced, "reduced")


def test_device_tile_index_matches_host():
    """The segment table the device builds (with its warp-scanned tile index) against the
    oracle's layout: the same (bucket, shard, lo, hi) rows, and each segment's first tile
    = the running count of the kTileElems cells the segments before it overlap."""
    for wl in list(reduced_workloads().values()) + list(full_workloads().values()):
        lay = _layout(wl)
        dev = lay.device_segments()
        segs = np.array(S.oracle_layout(wl).segments, dtype=np.int64).reshape(-1, 4)
        T = lay.tile_elems
        assert np.array_equal(dev[:-1, :4], segs)
        counts = [-(-hi // T) - lo // T for _, _, lo, hi in segs]
        assert list(dev[:-1, 4]) == list(np.cumsum([0] + counts)[:-1])
        assert dev[-1, 4] == lay.n_tiles == sum(counts)


# ------------------------------------------------------------- edge cases

def _edge(tensors, N, stage, B, A, steps=2, units=(), L=1024.0, **kw):
    return Workload(name="edge", description="edge", tensors=tuple(tensors), units=tuple(units), n_ranks=N,
                    stage=stage, bucket_elems=B, steps=steps, loss_scale=L, pad_align=A, **kw)


EDGES = {
    "ring3_trace": _edge([3], 3, 1, 0, 1),
    "one_rank": _edge([10_001], 1, 1, 999, 8),
    "two_ranks_unaligned": _edge([4097, 3, 7, 12_289], 2, 2, 37, 1),
    "five_ranks": _edge([77_777], 5, 0, 9_999, 1),
    "one_elem_buckets": _edge([301], 4, 2, 1, 1),
    "seven_elem_buckets": _edge([5_000], 6, 3, 7, 1, units=()),
    "seventeen_ranks_runtime_n": _edge([33_333, 1, 2], 17, 2, 4_111, 4, heavy_frac=0.05, heavy_mult=100.0),
    "stage3_units_unaligned": _edge([13, 4099, 8190, 5], 3, 3, 1_000, 1, units=(0, 1, 3)),
    "ddp_many_tiles": _edge([3 * 4096 * 148 + 5], 3, 0, 100_003, 128, m_sigma=1e-4, v_sigma=1e-6),
}


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("key", list(EDGES))
def test_edge_cases(key, impl):
    wl = EDGES[key]
    ref, _ = _oracle(wl)
    lay = _layout(wl, impl)
    b = _bufs(lay, wl, guard=True)
    _run(lay, wl, b, wl.steps)
    _check_full(wl, lay, b, ref)


def test_padded_rank_stride():
    wl = _edge([50_000], 4, 1, 7_000, 128)
    ref, _ = _oracle(wl)
    lay = _layout(wl)
    b = _bufs(lay, wl, rank_stride=lay.padded + 4096)
    _run(lay, wl, b, wl.steps)
    _check_full(wl, lay, b, ref)


def test_empty_layout_is_noop():
    lay = zs.Layout([], 4, 2, 100).to_device()
    zs.step(lay, 0, 0, 0, 0, 0, 0, zs.AdamW(), rank_stride=0)
    zs.reduce_scatter(lay, -1, 0, 0, rank_stride=0)
    zs.allgather(lay, -1, 0, 0)
    zs.get_error(lay)


def test_order_probe_on_gpu():
    # chunk k: ranks k, k+1 hold 2^-24, rank k+2 holds 1: only the ring order k, k+1, k+2
    # gives 1 + 2^-23
    lay = zs.Layout([3], 3, 1, 0, 1).to_device()
    g = np.zeros((3, 8), np.uint16)
    for k in range(3):
        g[k, k] = 1
        g[(k + 1) % 3, k] = 1
        g[(k + 2) % 3, k] = 0x3C00
    gd = torch.from_numpy(g.view(np.int16)).cuda()
    red = torch.zeros(8, dtype=torch.float32, device="cuda")
    zs.reduce_scatter(lay, -1, gd, red)
    assert np.all(_np(red)[:3] == np.float32(1) + np.float32(2 ** -23))


def test_nonfinite_counts_per_bucket():
    wl = _edge([30_000], 4, 2, 7_001, 8)
    olay = S.oracle_layout(wl)
    P = olay.padded
    g = np.zeros((4, P), np.uint16)
    marks = {3: 0x7C00, 7_000: 0xFC00, 7_001: 0x7E00, 22_222: 0x7C00, 29_999: 0x7C00}
    for i, bits in marks.items():
        g[i % 4, i] = bits
    g[0, 29_999] = 0xFC00
    master = np.zeros(P, np.float32)
    ref = oracle.run_steps(olay, 2, g, master, master, master, S.hyper(wl), 1)
    lay = _layout(wl)
    gd = torch.from_numpy(g.view(np.int16)).cuda()
    bufs = [torch.zeros(P, dtype=torch.float32, device="cuda") for _ in range(3)]
    p16 = torch.zeros(P, dtype=torch.int16, device="cuda")
    nf = torch.zeros(lay.n_buckets, dtype=torch.int32, device="cuda")
    zs.step(lay, gd, *bufs, None, p16, _hp(wl, 1), nonfinite=nf)
    assert list(_np(nf)) == list(ref.nonfinite)
    assert sum(ref.nonfinite) == len(marks)
    S.assert_f16_ulp(_np(p16), ref.p16_full, "p16")


@pytest.mark.parametrize("impl", IMPLS)
def test_zero_and_signed_zero_operands(impl):
    """Exact zeros take the kernels' shortcut around the square root and the divisions:
    zero gradients with zero moments (untouched rows), gradients of -0, moments of -0,
    zero gradients with warm moments, and eps = 0 (where 0 / 0 must stay NaN), for every
    step against the oracle bit for bit."""
    wl = _edge([40_000, 9_001], 4, 2, 10_007, 8, steps=3, m_sigma=1e-4, v_sigma=1e-6)
    olay = S.oracle_layout(wl)
    P = olay.padded
    g, master, m, v = S.host_inputs(wl, P)
    g[:, :12_000] = 0                                   # untouched rows: zero gradient, zero moments
    m[:12_000] = 0
    v[:12_000] = 0
    g[:, 12_000:14_000] = 0x8000                        # -0 gradients, warm moments
    g[:, 14_000:16_000] = 0x8000                        # -0 gradients, -0 first moment, zero second
    m[14_000:16_000] = -0.0
    v[14_000:16_000] = 0
    g[1, 16_000:18_000] = 0x8000                        # one rank's -0 among finite gradients
    g[:, 18_000:20_000] = 0                             # zero gradient, warm moments
    for eps in (1e-8, 0.0):
        w = wl.with_(eps=eps)
        ref = oracle.run_steps(olay, w.stage, g, master, m, v, S.hyper(w), w.steps)
        lay = _layout(w, impl)
        b = dict(g=torch.from_numpy(g.view(np.int16)).cuda(), master=torch.from_numpy(master).cuda(),
                 m=torch.from_numpy(m).cuda(), v=torch.from_numpy(v).cuda(),
                 p16_shard=torch.zeros(P, dtype=torch.int16, device="cuda"),
                 p16_full=torch.zeros(P, dtype=torch.int16, device="cuda"),
                 nonfinite=torch.zeros(lay.n_buckets, dtype=torch.int32, device="cuda"))
        for t in range(1, w.steps + 1):
            b["nonfinite"].zero_()
            zs.step(lay, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"], _hp(w, t),
                    nonfinite=b["nonfinite"])
        zs.get_error(lay)
        for k, want in (("master", ref.master), ("m", ref.m), ("v", ref.v), ("p16_full", ref.p16_full)):
            S.assert_bits_equal(_np(b[k]), want, k, any_nan=True)
        if eps == 0.0:
            assert np.isnan(ref.master[:12_000]).all()     # 0 / (0 + 0): the shortcut must not hide it
        assert np.signbit(ref.m[14_000:16_000]).all() and not ref.m[14_000:16_000].any()


def test_bad_arguments_rejected():
    wl = _edge([10_000], 2, 1, 1_000, 8)
    lay = _layout(wl)
    b = _bufs(lay, wl)
    with pytest.raises(zs.ZeroError) as e:
        zs.step(lay, b["g"], b["master"], b["m"], b["v"], None, b["p16_full"], _hp(wl, 0))
    assert e.value.status == 1
    with pytest.raises(zs.ZeroError) as e:
        zs.step(lay, b["g"], b["master"][1:], b["m"], b["v"], None, b["p16_full"], _hp(wl, 1))
    assert e.value.status == 2
    with pytest.raises(zs.ZeroError) as e:
        zs.step(lay, b["g"], b["master"], b["m"], b["v"], None, b["p16_full"], _hp(wl, 1),
                rank_stride=lay.padded - 8)
    assert e.value.status == 1
    with pytest.raises(zs.ZeroError):
        zs.reduce_scatter(lay, lay.n_buckets, b["g"], b["master"])
    with pytest.raises(zs.ZeroError):
        zs.allgather(lay, 5, b["p16_shard"], b["p16_full"])
    with pytest.raises(zs.ZeroError):
        zs.step(lay, b["g"], b["master"], b["m"], b["v"], None, b["p16_full"],
                zs.AdamW(loss_scale=0.0, step=1))


@pytest.mark.parametrize("impl", IMPLS)
def test_host_buffer_step_matches_oracle(impl):
    """zero_step_host: gradients from pinned host memory, fp16 parameters back to pinned
    host memory; the device state and the host parameters equal the oracle's."""
    for key in ("flat1p3b_n4_zero1", "llama3b_n8_zero3", "ragged2000_n16_zero2"):
        wl = reduced_workloads()[key]
        ref, olay = _oracle(wl, 2)
        lay = _layout(wl, impl)
        b = _bufs(lay, wl)
        g_host = torch.from_numpy(S.host_inputs(wl, olay.padded)[0].view(np.int16))
        pad = b["g"].shape[1] - g_host.shape[1]
        g_host = torch.nn.functional.pad(g_host, (0, pad)).contiguous().pin_memory()
        b["g"].zero_()
        p16_host = torch.zeros(lay.padded, dtype=torch.int16).pin_memory()
        for t in range(1, 3):
            zs.step_host(lay, g_host, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"],
                         p16_host, _hp(wl, t))
        torch.cuda.synchronize()
        S.assert_state_matches_oracle(wl, b, ref, key + ": ")
        S.assert_bits_equal(p16_host.numpy().view(np.uint16), ref.p16_full, key + ": p16_host")


# ------------------------------------------------------------- full size, sampled

@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("key", list(full_workloads()))
def test_full_size_sampled(key, impl):
    wl = full_workloads()[key]
    olay = S.oracle_layout(wl)
    lay = _layout(wl, impl)
    b = _bufs(lay, wl)
    _run(lay, wl, b, wl.steps)
    idx = S.sample_indices(olay)
    it = torch.from_numpy(idx).cuda()
    red_ref, master, m, v, p16 = S.sampled_oracle(wl, olay, idx, wl.steps)
    got = {k: _np(b[k][it]) for k in ("master", "m", "v", "p16_full", "p16_shard")}
    S.assert_f32_close(got["master"], master, "master")
    S.assert_f32_close(got["m"], m, "m")
    S.assert_f32_close(got["v"], v, "v")
    S.assert_f16_ulp(got["p16_full"], p16, "p16_full")
    S.assert_bits_equal(got["master"], master, "master")
    S.assert_bits_equal(got["m"], m, "m")
    S.assert_bits_equal(got["v"], v, "v")
    S.assert_bits_equal(got["p16_full"], p16, "p16_full")
    if wl.stage == 3:
        S.assert_bits_equal(got["p16_shard"], p16, "p16_shard")
    assert int(b["nonfinite"].sum()) == 0
    # ring sums at the sampled indices
    del b["m"], b["v"], b["p16_shard"]
    red = torch.empty(lay.padded, dtype=torch.float32, device="cuda")
    zs.reduce_scatter(lay, -1, b["g"], red)
    S.assert_bits_equal(_np(red[it]), red_ref, "reduced")
    # the padding stayed zero
    assert int(torch.count_nonzero(b["p16_full"][lay.psi:])) == 0
    assert int(torch.count_nonzero(b["master"][lay.psi:])) == 0


@pytest.mark.parametrize("key", ["flat1p3b_n4_zero1", "ragged2000_n16_zero2"])
def test_full_size_overlapped_sampled(key):
    """zero_step_overlapped at full size (the flat list's 27 buckets of 5*10^7, each its own
    launch; the ragged list's 490 buckets of 10^6, coalesced into launches of >= 2^24
    elements), every bucket's event recorded on a producer stream, through the plan
    tuner's first calls: the oracle's state at sampled elements, bit for bit."""
    wl = full_workloads()[key]
    olay = S.oracle_layout(wl)
    lay = _layout(wl, zs.IMPL_AUTO)
    b = _bufs(lay, wl)
    producer, consumer = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    for t in range(1, wl.steps + 1):
        ready = [torch.cuda.Event() for _ in range(lay.n_buckets)]
        for e in ready:
            e.record(producer)
        b["nonfinite"].zero_()
        torch.cuda.synchronize()
        zs.step_overlapped(lay, ready, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"],
                           _hp(wl, t), nonfinite=b["nonfinite"], stream=consumer)
        torch.cuda.synchronize()
    zs.get_error(lay)
    idx = S.sample_indices(olay)
    it = torch.from_numpy(idx).cuda()
    _, master, m, v, p16 = S.sampled_oracle(wl, olay, idx, wl.steps)
    for name, want in (("master", master), ("m", m), ("v", v), ("p16_full", p16)):
        S.assert_bits_equal(_np(b[name][it]), want, name)
    assert int(b["nonfinite"].sum()) == 0


@pytest.mark.parametrize("impl", IMPLS)
def test_full_size_dynamic_commit_sampled(impl):
    """zero_step_dynamic_commit at full size (flat list, two state sets and two fp16
    buffers of 1.3*10^9): with a scale that never overflows here and a window longer than
    the run, every step applies at the workload's loss scale, so after each commit the
    current set equals the oracle's plain steps at sampled elements, bit for bit."""
    wl = full_workloads()["flat1p3b_n4_zero1"]
    steps = 3
    olay = S.oracle_layout(wl)
    lay = _layout(wl, impl)
    P = lay.padded
    g, master, m, v = S.device_inputs(wl, P)
    sets = [[master, m, v], [torch.empty_like(master), torch.empty_like(m), torch.empty_like(v)]]
    p16s = [torch.zeros(P, dtype=torch.int16, device="cuda"), torch.zeros(P, dtype=torch.int16, device="cuda")]
    nonfinite = torch.zeros(max(1, lay.n_buckets), dtype=torch.int32, device="cuda")
    scaler = zs.LossScaler(wl.loss_scale, window=1 << 40)
    for t in range(1, steps + 1):
        assert zs.step_dynamic_commit(lay, g, sets[0], sets[1], p16s[1], p16s[1], _hp(wl, t), scaler, nonfinite)
        sets.reverse()
        p16s.reverse()
    zs.get_error(lay)
    torch.cuda.synchronize()
    assert scaler.scale == wl.loss_scale
    idx = S.sample_indices(olay)
    it = torch.from_numpy(idx).cuda()
    _, want_master, want_m, want_v, want_p16 = S.sampled_oracle(wl, olay, idx, steps)
    for name, got, want in (("master", sets[0][0], want_master), ("m", sets[0][1], want_m),
                            ("v", sets[0][2], want_v), ("p16", p16s[0], want_p16)):
        S.assert_bits_equal(_np(got[it]), want, name)


@pytest.mark.parametrize("impl", IMPLS)
def test_flat_buffer_beyond_2_32_elements(impl):
    """ψ just above 2^32 (N=2, full fp32 state: 86 GB on the device): element indices,
    byte offsets and tile numbers past 32 bits, sampled against the oracle, including
    every element around 2^31 and 2^32 and the shard edge."""
    wl = Workload(name="beyond32", description="beyond 2^32", tensors=((1 << 32) + 4097,), units=(), n_ranks=2,
                  stage=1, bucket_elems=1_000_000_007, steps=2, loss_scale=1024.0, m_sigma=1e-4, v_sigma=1e-6)
    olay = S.oracle_layout(wl)
    lay = _layout(wl, impl)
    assert lay.padded > (1 << 32) and lay.n_tiles > (1 << 20)
    b = _bufs(lay, wl)
    _run(lay, wl, b, wl.steps)
    near = [c + d for c in (1 << 31, 1 << 32, olay.shard) for d in range(-9, 10)]
    idx = np.unique(np.concatenate([S.sample_indices(olay), np.array(near, np.int64)]))
    it = torch.from_numpy(idx).cuda()
    red_ref, master, m, v, p16 = S.sampled_oracle(wl, olay, idx, wl.steps)
    for k, want in (("master", master), ("m", m), ("v", v), ("p16_full", p16)):
        S.assert_bits_equal(_np(b[k][it]), want, k)
    assert int(b["nonfinite"].sum()) == 0
    del b["m"], b["v"], b["p16_shard"]
    red = torch.empty(lay.padded, dtype=torch.float32, device="cuda")
    zs.reduce_scatter(lay, -1, b["g"], red)
    S.assert_bits_equal(_np(red[it]), red_ref, "reduced")
    assert int(torch.count_nonzero(b["p16_full"][lay.psi:])) == 0


def test_bulk_pipeline_bounded_wait_reports_timeout():
    """The bulk pipeline's waits are bounded: with its first chunk never posted, the
    consumers' wait expires after 1 ms, the kernel drains and returns, the host reads
    ZERO_ERR_TIMEOUT, and the same context then runs a correct step."""
    wl = reduced_workloads()["flat1p3b_n4_zero1"]
    ref, _ = _oracle(wl, steps=1)
    lay = _layout(wl, zs.IMPL_BULK)
    b = _bufs(lay, wl)
    lay.debug_set_wait(1_000_000, skip_first_fill=1)
    zs.step(lay, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"], _hp(wl, 1))
    with pytest.raises(zs.ZeroError) as e:
        zs.get_error(lay)
    assert e.value.status == 5
    zs.get_error(lay)                        # the word was cleared
    lay.debug_set_wait(2_000_000_000, skip_first_fill=0)
    b = _bufs(lay, wl)
    _run(lay, wl, b, 1)
    _check_full(wl, lay, b, ref)


@pytest.mark.parametrize("key", ["flat1p3b_n4_zero1", "llama3b_n8_zero3"])
def test_checkpoint_resume_matches_oracle(key):
    """The optimizer state is the caller's buffers: copying them to host memory after two
    steps, wiping the device buffers and a fresh layout, restoring, and running two more
    steps gives the oracle's uninterrupted four-step result (the library keeps no state
    of its own)."""
    wl = reduced_workloads()[key]
    ref, _ = _oracle(wl, 4)
    lay = _layout(wl, zs.IMPL_BULK)
    b = _bufs(lay, wl)
    for t in (1, 2):
        zs.step(lay, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"], _hp(wl, t))
    torch.cuda.synchronize()
    saved = {k: b[k].cpu().clone() for k in ("master", "m", "v", "p16_shard", "p16_full")}
    for k in saved:
        b[k].fill_(7)
    lay.close()
    lay2 = _layout(wl, zs.IMPL_BULK)
    for k, x in saved.items():
        b[k].copy_(x)
    for t in (3, 4):
        zs.step(lay2, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"], _hp(wl, t))
    torch.cuda.synchronize()
    S.assert_state_matches_oracle(wl, b, ref)
