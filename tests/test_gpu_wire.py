"""GPU parity of the fp16-wire ring and of dynamic loss scaling against the oracle.

- every reduced workload with partials travelling as fp16: ring sums, master, moments and
  fp16 parameters bit-exact (both fused implementations);
- a partial sum that overflows fp16 on the wire but not in fp32, counted per bucket;
- a run under dynamic loss scaling that starts at a scale whose gradients overflow:
  the sequence of skipped / applied steps, the scales used, the final scaler state and
  the final optimizer state all equal the oracle's (fp32 and fp16 wire);
- one full-size workload with the fp16 wire, sampled.
"""
import numpy as np
import pytest

import oracle
import seeded_inputs as si
from seeded_inputs.workloads import full_workloads, reduced_workloads
import zero_sharded_optimizer_ring_b200 as zs
import support as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _hp(wl, t, scale=None):
    return zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, scale or wl.loss_scale, t)


def _layout(wl, impl, wire=True):
    lay = zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units),
                    wire_fp16=wire).to_device()
    lay.set_impl(impl)
    return lay


def _np(t):
    a = t.cpu().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a


def _bufs(wl, P):
    g, master, m, v = S.device_inputs(wl, P)
    return dict(g=g, master=master, m=m, v=v, p16_shard=torch.zeros(P, dtype=torch.int16, device="cuda"),
                p16_full=torch.zeros(P, dtype=torch.int16, device="cuda"),
                nonfinite=torch.zeros(4096, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("impl", [zs.IMPL_REGISTER, zs.IMPL_BULK])
@pytest.mark.parametrize("key", list(reduced_workloads()))
def test_wire_matches_oracle(key, impl):
    wl = reduced_workloads()[key]
    olay = S.oracle_layout(wl)
    g, master, m, v = S.host_inputs(wl, olay.padded)
    ref = oracle.run_steps(olay, wl.stage, g, master, m, v, S.hyper(wl), wl.steps, wire16=True)
    lay = _layout(wl, impl)
    b = _bufs(wl, lay.padded)
    for t in range(1, wl.steps + 1):
        b["nonfinite"].zero_()
        zs.step(lay, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"], _hp(wl, t),
                nonfinite=b["nonfinite"])
    zs.get_error(lay)
    for k, want in (("master", ref.master), ("m", ref.m), ("v", ref.v), ("p16_full", ref.p16_full)):
        S.assert_bits_equal(_np(b[k]), want, k)
    assert list(_np(b["nonfinite"])[:lay.n_buckets]) == list(ref.nonfinite)
    red = torch.zeros(lay.padded, dtype=torch.float32, device="cuda")
    zs.reduce_scatter(lay, -1, b["g"], red)
    S.assert_bits_equal(_np(red), ref.reduced, "reduced")


def test_wire_overflow_counted_where_fp32_is_finite():
    wl = reduced_workloads()["flat1p3b_n4_zero1"].with_(tensors=(20_000,), bucket_elems=3_001)
    olay = S.oracle_layout(wl)
    P = olay.padded
    rng = np.random.default_rng(3)
    x = rng.uniform(-1.0, 1.0, (4, P))
    x[:, ::97] = 30000.0                       # four ranks of 30000: the wire overflows
    x[:, 20_000:] = 0
    g = np.ascontiguousarray(x.astype(np.float16).view(np.uint16))
    gd = torch.from_numpy(g.view(np.int16)).cuda()
    zero = np.zeros(P, np.float32)
    for wire in (False, True):
        ref = oracle.run_steps(olay, 1, g, zero, zero, zero, S.hyper(wl), 1, wire16=wire)
        for impl in (zs.IMPL_REGISTER, zs.IMPL_BULK):
            lay = _layout(wl, impl, wire)
            st = [torch.zeros(P, dtype=torch.float32, device="cuda") for _ in range(3)]
            p16 = torch.zeros(P, dtype=torch.int16, device="cuda")
            nf = torch.zeros(lay.n_buckets, dtype=torch.int32, device="cuda")
            zs.step(lay, gd, *st, None, p16, _hp(wl, 1), nonfinite=nf)
            assert list(_np(nf)) == list(ref.nonfinite)
            assert (sum(ref.nonfinite) > 0) == wire
            S.assert_f16_ulp(_np(p16), ref.p16_full, "p16")


@pytest.mark.parametrize("wire", [False, True])
def test_dynamic_loss_scaling_matches_oracle(wire):
    wl = reduced_workloads()["flat1p3b_n4_zero1"]
    olay = S.oracle_layout(wl)
    P, psi = olay.padded, wl.psi
    _, master, m, v = S.host_inputs(wl, P)
    start, steps = 2.0 ** 24, 12

    def grads_at(scale, i):
        return si.fill_grads(wl.n_ranks, P, psi, wl.seed + i, wl.grad_sigma, scale)

    osc = oracle.LossScaler(start, window=3)
    ref, trace = oracle.run_steps_dynamic(olay, wl.stage, grads_at, master, m, v, S.hyper(wl), steps, osc,
                                          wire16=wire)
    assert any(o for _, o, _ in trace) and not all(o for _, o, _ in trace)

    lay = _layout(wl, zs.IMPL_BULK, wire)
    b = _bufs(wl, P)
    red = torch.zeros(P, dtype=torch.float32, device="cuda")
    sc = zs.LossScaler(start, window=3)
    got = []
    for i in range(steps):
        used = sc.scale
        si.fill_grads_cuda(b["g"], psi, wl.seed + i, wl.grad_sigma, used)
        applied = zs.step_dynamic(lay, b["g"], red, b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"],
                                  _hp(wl, 1), sc, b["nonfinite"])
        got.append((used, not applied, sc.step if applied else 0))
    torch.cuda.synchronize()
    assert got == trace
    assert (sc.scale, sc.clean_steps, sc.step, sc.skipped) == (osc.scale, osc.clean_steps, osc.step, osc.skipped)
    for k, want in (("master", ref.master), ("m", ref.m), ("v", ref.v), ("p16_full", ref.p16_full)):
        S.assert_bits_equal(_np(b[k]), want, k)


def _commit_cases():
    red = reduced_workloads()
    cases = [(k, w, impl) for k in ("flat1p3b_n4_zero1", "llama3b_n8_zero3", "ragged2000_n16_zero2")
             for w in (False, True) for impl in (zs.IMPL_BULK, zs.IMPL_REGISTER)]
    return cases + [("ragged_n17", w, zs.IMPL_AUTO) for w in (False, True)]


def _commit_workload(key):
    if key == "ragged_n17":                 # no pipeline specialisation: register streaming
        return reduced_workloads()["ragged2000_n16_zero2"].with_(n_ranks=17)
    return reduced_workloads()[key]


@pytest.mark.parametrize("key,wire,impl", _commit_cases())
def test_dynamic_commit_matches_oracle(key, wire, impl):
    """The two-phase commit: state read from one buffer set, written to the other, the
    sets swapped only on applied steps.  Same skip / apply trace, scaler and final state
    as the oracle's dynamic run; a skipped step leaves the current set and p16 untouched."""
    wl = _commit_workload(key)
    olay = S.oracle_layout(wl)
    P, psi = olay.padded, wl.psi
    _, master, m, v = S.host_inputs(wl, P)
    start, steps = 2.0 ** 24, 10

    def grads_at(scale, i):
        return si.fill_grads(wl.n_ranks, P, psi, wl.seed + i, wl.grad_sigma, scale)

    osc = oracle.LossScaler(start, window=3)
    ref, trace = oracle.run_steps_dynamic(olay, wl.stage, grads_at, master, m, v, S.hyper(wl), steps, osc,
                                          wire16=wire)
    assert any(o for _, o, _ in trace) and not all(o for _, o, _ in trace)

    lay = _layout(wl, impl, wire)
    b = _bufs(wl, P)
    cur = (b["master"], b["m"], b["v"])
    nxt = tuple(torch.full_like(x, float("nan")) for x in cur)
    # stages 0-2: two full fp16 buffers take turns; stage 3: two shard-written buffers
    # take turns and p16_full receives the gather of an applied step
    p16_cur = b["p16_shard"] if wl.stage == 3 else b["p16_full"]
    p16_nxt = torch.zeros_like(p16_cur)
    gathered = b["p16_full"] if wl.stage == 3 else None
    sc = zs.LossScaler(start, window=3)
    got = []
    for i in range(steps):
        used = sc.scale
        si.fill_grads_cuda(b["g"], psi, wl.seed + i, wl.grad_sigma, used)
        kept = list(cur) + [p16_cur] + ([gathered] if gathered is not None else [])
        before = [x.clone() for x in kept]
        applied = zs.step_dynamic_commit(lay, b["g"], cur, nxt, p16_nxt, gathered, _hp(wl, 1), sc,
                                         b["nonfinite"])
        got.append((used, not applied, sc.step if applied else 0))
        if applied:
            cur, nxt = nxt, cur
            p16_cur, p16_nxt = p16_nxt, p16_cur
        else:
            for x, y in zip(kept, before):
                S.assert_bits_equal(_np(x), _np(y), "untouched on a skipped step")
    torch.cuda.synchronize()
    zs.get_error(lay)
    assert got == trace
    assert (sc.scale, sc.clean_steps, sc.step, sc.skipped) == (osc.scale, osc.clean_steps, osc.step, osc.skipped)
    for name, x, want in (("master", cur[0], ref.master), ("m", cur[1], ref.m), ("v", cur[2], ref.v),
                          ("p16_full", gathered if wl.stage == 3 else p16_cur, ref.p16_full)):
        S.assert_bits_equal(_np(x), want, name)


def test_dynamic_commit_rejects_overlapping_sets():
    wl = reduced_workloads()["flat1p3b_n4_zero1"]
    lay = _layout(wl, zs.IMPL_BULK, False)
    b = _bufs(wl, lay.padded)
    st = (b["master"], b["m"], b["v"])
    sc = zs.LossScaler(1024.0)
    for out in (st, (b["master"], torch.empty_like(b["m"]), torch.empty_like(b["v"]))):
        with pytest.raises(zs.ZeroError) as e:
            zs.step_dynamic_commit(lay, b["g"], st, out, b["p16_shard"], None, _hp(wl, 1), sc, b["nonfinite"])
        assert e.value.status == 1
    assert (sc.step, sc.skipped) == (0, 0)


def test_wire_full_size_sampled():
    wl = full_workloads()["flat1p3b_n4_zero1"]
    olay = S.oracle_layout(wl)
    lay = _layout(wl, zs.IMPL_BULK)
    b = _bufs(wl, lay.padded)
    steps = 3
    for t in range(1, steps + 1):
        zs.step(lay, b["g"], b["master"], b["m"], b["v"], None, b["p16_full"], _hp(wl, t))
    torch.cuda.synchronize()
    idx = S.sample_indices(olay)
    it = torch.from_numpy(idx).cuda()
    psi = wl.psi
    g = si.gather_grads(idx, wl.n_ranks, psi, wl.seed, wl.grad_sigma, wl.loss_scale)
    master = si.gather_f32(idx, psi, wl.seed, si.STREAM_MASTER, wl.master_sigma)
    m = si.gather_f32(idx, psi, wl.seed, si.STREAM_M, wl.m_sigma)
    v = si.gather_f32(idx, psi, wl.seed, si.STREAM_V, wl.v_sigma, True)
    sc = np.stack([oracle.adamw_scalars(wl.n_ranks, S.hyper(wl), t) for t in range(1, steps + 1)])
    _, p16 = oracle.sampled(g, idx // olay.shard, steps, sc, master, m, v, wire16=True)
    S.assert_bits_equal(_np(b["master"][it]), master, "master")
    S.assert_bits_equal(_np(b["m"][it]), m, "m")
    S.assert_bits_equal(_np(b["v"][it]), v, "v")
    S.assert_bits_equal(_np(b["p16_full"][it]), p16, "p16_full")
