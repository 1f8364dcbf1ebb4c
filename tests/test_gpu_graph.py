"""The step with device-resident scalars, plain and captured once in a CUDA graph.

zero_step_device_scalars reads the step's nine fp32 scalars from device memory when its
kernels run, so one capture of it (with a copy of the scalars from page-locked host
memory in front) can be replayed for every step.  Every replay must give the CPU
oracle's state after the same number of steps, bit for bit; so must the uncaptured call,
in both implementations.  (zero_step_scalars_fill is checked against the oracle's
scalars on the CPU, in test_abi_host.py.)
"""
import pytest

from seeded_inputs.workloads import reduced_workloads
import zero_sharded_optimizer_ring_b200 as zs
import support as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _hp(wl, t):
    return zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale, t)


def _setup(wl, impl=zs.IMPL_AUTO):
    lay = zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align,
                    list(wl.units)).to_device()
    lay.set_impl(impl)
    P = lay.padded
    g, master, m, v = S.device_inputs(wl, P)
    b = dict(g=g, master=master, m=m, v=v, p16_shard=torch.zeros(P, dtype=torch.int16, device="cuda"),
             p16_full=torch.zeros(P, dtype=torch.int16, device="cuda"),
             nonfinite=torch.zeros(max(1, lay.n_buckets), dtype=torch.int32, device="cuda"))
    return lay, b


def _call(lay, b, scalars_dev, stream=None):
    zs.step_device_scalars(lay, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"], scalars_dev,
                           nonfinite=b["nonfinite"], stream=stream)


@pytest.mark.parametrize("impl", [zs.IMPL_REGISTER, zs.IMPL_BULK])
@pytest.mark.parametrize("key", list(reduced_workloads()))
def test_device_scalars_step_matches_oracle(key, impl):
    wl = reduced_workloads()[key]
    ref, _ = S.oracle_run(wl)
    lay, b = _setup(wl, impl)
    scalars = torch.empty(9, dtype=torch.float32, device="cuda")
    for t in range(1, wl.steps + 1):
        scalars.copy_(torch.from_numpy(zs.step_scalars(lay, _hp(wl, t))))
        b["nonfinite"].zero_()
        _call(lay, b, scalars)
    zs.get_error(lay)
    torch.cuda.synchronize()
    S.assert_state_matches_oracle(wl, b, ref)
    assert list(S.to_np(b["nonfinite"])[:lay.n_buckets]) == list(ref.nonfinite)


@pytest.mark.parametrize("key", ["ring3_psi1m_zero1", "flat1p3b_n4_zero1", "llama3b_n8_zero3",
                                 "ragged2000_n16_zero2"])
def test_step_captured_in_a_cuda_graph_matches_oracle(key):
    """One capture (scalar copy from pinned host memory + the step), replayed once per
    step with the host copy rewritten between replays."""
    wl = reduced_workloads()[key]
    ref, _ = S.oracle_run(wl)
    lay, b = _setup(wl)
    host = torch.zeros(9, dtype=torch.float32).pin_memory()
    scalars = torch.zeros(9, dtype=torch.float32, device="cuda")
    # load the kernels outside the capture, on copies that the test then discards
    scratch = {k: x.clone() for k, x in b.items()}
    scalars.copy_(torch.from_numpy(zs.step_scalars(lay, _hp(wl, 1))))
    _call(lay, scratch, scalars)
    torch.cuda.synchronize()
    del scratch
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.graph(graph, stream=side):
        scalars.copy_(host, non_blocking=True)
        _call(lay, b, scalars)
    for t in range(1, wl.steps + 1):
        host.copy_(torch.from_numpy(zs.step_scalars(lay, _hp(wl, t))))
        graph.replay()
        torch.cuda.synchronize()                     # the host copy is read when the replay runs
    zs.get_error(lay)
    S.assert_state_matches_oracle(wl, b, ref)
    del graph


def test_device_scalars_argument_checks():
    wl = reduced_workloads()["flat1p3b_n4_zero1"]
    lay, b = _setup(wl)
    scalars = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(zs.ZeroError) as e:
        _call(lay, b, None)
    assert e.value.status == 1
    with pytest.raises(zs.ZeroError) as e:
        _call(lay, b, scalars.view(torch.uint8)[1:].data_ptr())      # not 4-byte aligned
    assert e.value.status == 2
