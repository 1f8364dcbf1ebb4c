"""ZeRO-3 per-layer gathers: zero_gather_unit and the prefetching schedule.

Every unit gathered into its own buffer equals its range of the shard buffer, bit for bit
(aligned and unaligned unit starts).  Under the prefetching schedule, each layer's
"compute" (a deliberate delay, then a copy of the gathered buffer to the unit's place in
an output buffer) must see its own unit's parameters: a slot overwritten before its
layer finished would show up as a mismatch.
"""
import numpy as np
import pytest

from seeded_inputs.workloads import reduced_workloads
import zero_sharded_optimizer_ring_b200 as zs
from zero_sharded_optimizer_ring_b200.schedule import zero3_pass

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _setup(tensors, units, N=8):
    lay = zs.Layout(list(tensors), N, 3, 50_000, 1, list(units)).to_device()
    P = lay.padded
    shard = torch.randint(-30000, 30000, (P,), dtype=torch.int16, device="cuda")
    _, _, _, u = lay.tables()
    return lay, shard, u


@pytest.mark.parametrize("aligned", [True, False])
def test_gather_unit_equals_its_range(aligned):
    wl = reduced_workloads()["llama3b_n8_zero3"]
    tensors = list(wl.tensors) if aligned else [3] + list(wl.tensors)[1:]
    units = list(wl.units)
    lay, shard, u = _setup(tensors, units)
    assert aligned == all(lo % 8 == 0 for lo, _ in u)
    for k, (lo, hi) in enumerate(u):
        dst = torch.full((hi - lo + 16,), 7, dtype=torch.int16, device="cuda")
        zs.gather_unit(lay, k, shard, dst)
        torch.cuda.synchronize()
        assert torch.equal(dst[:hi - lo], shard[lo:hi])
        assert torch.all(dst[hi - lo:] == 7)


@pytest.mark.parametrize("n_slots", [1, 2, 3])
@pytest.mark.parametrize("backward", [False, True])
def test_prefetch_schedule_gives_each_layer_its_parameters(n_slots, backward):
    wl = reduced_workloads()["llama3b_n8_zero3"]
    lay, shard, u = _setup(wl.tensors, wl.units)
    width = int(max(hi - lo for lo, hi in u))
    slots = [torch.zeros(width, dtype=torch.int16, device="cuda") for _ in range(n_slots)]
    out = torch.zeros(lay.padded, dtype=torch.int16, device="cuda")
    order = list(range(lay.n_units))
    if backward:
        order.reverse()

    def compute(unit, buf):
        torch.cuda._sleep(200_000)                  # a slow layer: gathers run far ahead if allowed
        lo, hi = int(u[unit][0]), int(u[unit][1])
        out[lo:hi].copy_(buf[:hi - lo])

    gs, cs = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()                        # inputs written on the default stream
    zero3_pass(lay, shard, slots, order, compute, gs, cs)
    torch.cuda.synchronize()
    assert torch.equal(out, shard)
