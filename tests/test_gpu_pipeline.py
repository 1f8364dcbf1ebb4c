"""Bucket pipelining: the per-bucket step and the event-gated step against the oracle.

A simulated backward pass writes one bucket of gradients at a time, last bucket of the
flat buffer first (the order a backward pass completes them: rkmt.cn/news/44736 "DDP",
en.pswp.cn/web/84187 "DDP" buckets), on its own stream and records an event per bucket;
zero_step_overlapped runs each bucket's fused update on another stream as soon as its
event fires.  Every state buffer, the fp16 parameters and the per-bucket non-finite
counts must equal the CPU oracle's (oracle.run_steps) bit for bit.
"""
import pytest

from seeded_inputs.workloads import reduced_workloads
import seeded_inputs as si
import zero_sharded_optimizer_ring_b200 as zs
import support as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _hp(wl, t):
    return zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale, t)


def _setup(wl):
    lay = zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align,
                    list(wl.units)).to_device()
    P = lay.padded

    def bufs():
        g, master, m, v = S.device_inputs(wl, P)
        return dict(g=g, master=master, m=m, v=v,
                    p16_shard=torch.zeros(P, dtype=torch.int16, device="cuda"),
                    p16_full=torch.zeros(P, dtype=torch.int16, device="cuda"),
                    nonfinite=torch.zeros(max(1, lay.n_buckets), dtype=torch.int32, device="cuda"))
    return lay, bufs


def _check(wl, lay, b, ref):
    torch.cuda.synchronize()
    S.assert_state_matches_oracle(wl, b, ref)
    assert list(S.to_np(b["nonfinite"])[:lay.n_buckets]) == list(ref.nonfinite)


STEPS = 2


@pytest.mark.parametrize("key", list(reduced_workloads()))
@pytest.mark.parametrize("order", ["bucket", "reverse"])
def test_step_bucket_matches_oracle(key, order):
    wl = reduced_workloads()[key]
    ref, _ = S.oracle_run(wl, STEPS)
    lay, bufs = _setup(wl)
    b = bufs()
    seq = list(range(lay.n_buckets))
    if order == "reverse":
        seq.reverse()
    for t in range(1, STEPS + 1):
        b["nonfinite"].zero_()
        for bk in seq:
            zs.step_bucket(lay, bk, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"], _hp(wl, t),
                           nonfinite=b["nonfinite"])
        if wl.stage == 3:
            zs.allgather(lay, -1, b["p16_shard"], b["p16_full"])
    _check(wl, lay, b, ref)


@pytest.mark.parametrize("group", [None, 1, 3, 1000])
@pytest.mark.parametrize("key", ["flat1p3b_n4_zero1", "llama3b_n8_zero3", "ragged2000_n16_zero2"])
def test_overlapped_step_with_simulated_backward(key, group):
    wl = reduced_workloads()[key]
    ref, _ = S.oracle_run(wl, STEPS)
    lay, bufs = _setup(wl)
    b = bufs()
    _, buckets, _, _ = lay.tables()
    producer, consumer = torch.cuda.Stream(), torch.cuda.Stream()
    for t in range(1, STEPS + 1):
        torch.cuda.synchronize()
        b["g"].zero_()
        b["nonfinite"].zero_()
        torch.cuda.synchronize()
        ready = [torch.cuda.Event() for _ in range(lay.n_buckets)]
        for bk, (lo, hi) in enumerate(buckets):            # the backward: bucket 0 (the tail) first
            si.fill_grads_range_cuda(b["g"], int(lo), int(hi), wl.psi, wl.seed, wl.grad_sigma, wl.loss_scale,
                                     wl.heavy_frac, wl.heavy_mult, cuda_stream=producer.cuda_stream)
            ready[bk].record(producer)
        zs.step_overlapped(lay, ready, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"],
                           _hp(wl, t), nonfinite=b["nonfinite"], stream=consumer, group=group)
    zs.get_error(lay)
    _check(wl, lay, b, ref)


@pytest.mark.parametrize("wire", [False, True])
@pytest.mark.parametrize("impl", [zs.IMPL_REGISTER, zs.IMPL_BULK])
@pytest.mark.parametrize("key", ["flat1p3b_n4_zero1", "llama3b_n8_zero3", "ragged2000_n16_zero2"])
def test_overlapped_step_each_kernel_each_wire(key, impl, wire):
    """The overlapped step through each implementation, forced, with fp32 sums and with
    the fp16 wire, gradients arriving bucket by bucket: the oracle's state bit for bit
    (its fp16-wire run for the fp16 wire), per-bucket non-finite counts included."""
    import oracle
    wl = reduced_workloads()[key]
    olay = S.oracle_layout(wl)
    g, master, m, v = S.host_inputs(wl, olay.padded)
    ref = oracle.run_steps(olay, wl.stage, g, master, m, v, S.hyper(wl), STEPS, wire16=wire)
    lay = zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units),
                    wire_fp16=wire).to_device()
    lay.set_impl(impl)
    P = lay.padded
    gd, md, mm, vd = S.device_inputs(wl, P)
    b = dict(g=gd, master=md, m=mm, v=vd, p16_shard=torch.zeros(P, dtype=torch.int16, device="cuda"),
             p16_full=torch.zeros(P, dtype=torch.int16, device="cuda"),
             nonfinite=torch.zeros(max(1, lay.n_buckets), dtype=torch.int32, device="cuda"))
    _, buckets, _, _ = lay.tables()
    producer, consumer = torch.cuda.Stream(), torch.cuda.Stream()
    for t in range(1, STEPS + 1):
        torch.cuda.synchronize()
        b["g"].zero_()
        b["nonfinite"].zero_()
        torch.cuda.synchronize()
        ready = [torch.cuda.Event() for _ in range(lay.n_buckets)]
        for bk, (lo, hi) in enumerate(buckets):
            si.fill_grads_range_cuda(b["g"], int(lo), int(hi), wl.psi, wl.seed, wl.grad_sigma, wl.loss_scale,
                                     wl.heavy_frac, wl.heavy_mult, cuda_stream=producer.cuda_stream)
            ready[bk].record(producer)
        zs.step_overlapped(lay, ready, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"],
                           _hp(wl, t), nonfinite=b["nonfinite"], stream=consumer)
    zs.get_error(lay)
    _check(wl, lay, b, ref)


@pytest.mark.parametrize("key", ["flat1p3b_n4_zero1", "ragged2000_n16_zero2"])
def test_overlapped_grid_tuner_keeps_results(key):
    """With no cap set, the overlapped step times several launch plans over its first calls
    and then keeps the fastest; every call, whatever its plan, must give the oracle's
    result (14 steps: a warm-up, each of five plans timed twice, then the chosen one)."""
    wl = reduced_workloads()[key]
    steps = 14
    ref, _ = S.oracle_run(wl, steps)
    lay, bufs = _setup(wl)
    b = bufs()
    _, buckets, _, _ = lay.tables()
    producer, consumer = torch.cuda.Stream(), torch.cuda.Stream()
    for t in range(1, steps + 1):
        ready = [torch.cuda.Event() for _ in range(lay.n_buckets)]
        for bk in range(lay.n_buckets):
            ready[bk].record(producer)
        b["nonfinite"].zero_()
        torch.cuda.synchronize()
        zs.step_overlapped(lay, ready, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"],
                           _hp(wl, t), nonfinite=b["nonfinite"], stream=consumer, group=None if t % 2 else 2)
        torch.cuda.synchronize()                  # the tuner reads the call's events next time
    zs.get_error(lay)
    _check(wl, lay, b, ref)
    plan, means = lay.overlap_plan()
    assert 0 <= plan < zs._abi.OVERLAP_PLANS and len(means) == zs._abi.OVERLAP_PLANS
    assert all(x > 0 for x in means)                         # every plan timed, one kept
    assert means[plan] == min(means)


def test_overlapped_rejects_unrecorded_events():
    wl = reduced_workloads()["flat1p3b_n4_zero1"]
    lay, bufs = _setup(wl)
    b = bufs()
    with pytest.raises(ValueError):
        zs.step_overlapped(lay, [torch.cuda.Event() for _ in range(lay.n_buckets)], b["g"], b["master"], b["m"],
                           b["v"], None, b["p16_full"], _hp(wl, 1))
    with pytest.raises(zs.ZeroError):
        zs.step_bucket(lay, lay.n_buckets, b["g"], b["master"], b["m"], b["v"], None, b["p16_full"], _hp(wl, 1))
    ready = [torch.cuda.Event() for _ in range(lay.n_buckets)]
    for e in ready:
        e.record()
    with pytest.raises(zs.ZeroError) as err:
        zs.step_overlapped(lay, ready, b["g"], b["master"], b["m"], b["v"], None, b["p16_full"], _hp(wl, 1), group=0)
    assert err.value.status == 1
