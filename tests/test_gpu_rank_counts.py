"""GPU parity for every rank count the kernels specialise, and for counts they do not.

The fused step has one compiled variant per rank count: the bulk-copy pipeline for
N = 1..16 and one runtime-N pipeline instance for N = 17..64, the register-streaming
kernel for N = 1..8 and 16, and a runtime-N register kernel for all others. Each N runs a
small ragged layout (several tiles per shard, bucket and shard edges that are not
8-aligned for odd N) for two steps, in both implementations and with fp32 and fp16
partials on the wire, and must equal the oracle bit for bit. zero_step_ranks (one
gradient buffer per rank) is checked for N = 1..16 and for runtime-N counts up to 64.
"""
import numpy as np
import pytest

import oracle
from seeded_inputs.workloads import Workload
import zero_sharded_optimizer_ring_b200 as zs
import support as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

RANK_COUNTS = list(range(1, 21)) + [24, 32, 50, 51, 64, 65]


def _workload(N):
    # two full tiles per shard plus a ragged remainder; odd N pads to 1 element so that
    # shard (and so segment) edges fall inside 8-element vectors
    return Workload(name=f"ranks{N}", description="rank-count sweep",
                    tensors=(N * 2 * 4096 + 4099, 37, 1 + N), units=(), n_ranks=N, stage=(0, 1, 2, 3)[N % 4],
                    bucket_elems=3 * 4096 + 5, steps=2, loss_scale=1024.0, pad_align=1 if N % 2 else 8,
                    m_sigma=1e-4, v_sigma=1e-6, heavy_frac=0.01, heavy_mult=100.0)


def _hp(wl, t):
    return zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale, t)


def _np(t):
    a = t.cpu().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a


def _reference(wl, wire):
    olay = S.oracle_layout(wl)
    g, master, m, v = S.host_inputs(wl, olay.padded)
    return oracle.run_steps(olay, wl.stage, g, master, m, v, S.hyper(wl), wl.steps, wire16=wire)


def _check(wl, got, ref, n_buckets):
    for k, want in (("master", ref.master), ("m", ref.m), ("v", ref.v), ("p16_full", ref.p16_full)):
        S.assert_bits_equal(_np(got[k]), want, k)
    if wl.stage == 3:
        S.assert_bits_equal(_np(got["p16_shard"]), ref.p16_shard, "p16_shard")
    assert list(_np(got["nonfinite"])[:n_buckets]) == list(ref.nonfinite)


def _buffers(wl, P):
    g, master, m, v = S.device_inputs(wl, P)
    return g, dict(master=master, m=m, v=v, p16_shard=torch.zeros(P, dtype=torch.int16, device="cuda"),
                   p16_full=torch.zeros(P, dtype=torch.int16, device="cuda"),
                   nonfinite=torch.zeros(64, dtype=torch.int32, device="cuda"))


@pytest.fixture(autouse=True)
def _free():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("wire", [False, True])
@pytest.mark.parametrize("N", RANK_COUNTS)
def test_every_rank_count_both_kernels(N, wire):
    wl = _workload(N)
    ref = _reference(wl, wire)
    for impl in (zs.IMPL_REGISTER, zs.IMPL_BULK):
        lay = zs.Layout(list(wl.tensors), N, wl.stage, wl.bucket_elems, wl.pad_align, wire_fp16=wire).to_device()
        lay.set_impl(impl)
        assert lay.n_buckets <= 64
        g, b = _buffers(wl, lay.padded)
        for t in range(1, wl.steps + 1):
            b["nonfinite"].zero_()
            zs.step(lay, g, b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"], _hp(wl, t),
                    nonfinite=b["nonfinite"])
        zs.get_error(lay)
        _check(wl, b, ref, lay.n_buckets)
        # the reduce-scatter alone, in the same implementation (its reduce-only instances)
        red = torch.zeros(lay.padded, dtype=torch.float32, device="cuda")
        b["nonfinite"].zero_()
        zs.reduce_scatter(lay, -1, g, red, nonfinite=b["nonfinite"])
        zs.get_error(lay)
        S.assert_bits_equal(_np(red), ref.reduced, f"reduced, impl {impl}", any_nan=True)
        assert list(_np(b["nonfinite"])[:lay.n_buckets]) == list(ref.nonfinite)


@pytest.mark.parametrize("N", list(range(1, 18)) + [24, 33, 51, 64])
def test_step_ranks_every_pipeline_rank_count(N):
    wl = _workload(N)
    ref = _reference(wl, False)
    lay = zs.Layout(list(wl.tensors), N, wl.stage, wl.bucket_elems, wl.pad_align).to_device()
    g, b = _buffers(wl, lay.padded)
    ranks = [g[r].clone() for r in range(N)]                # one allocation per rank
    del g
    for t in range(1, wl.steps + 1):
        b["nonfinite"].zero_()
        zs.step_ranks(lay, ranks, b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"], _hp(wl, t),
                      nonfinite=b["nonfinite"])
    zs.get_error(lay)
    _check(wl, b, ref, lay.n_buckets)
