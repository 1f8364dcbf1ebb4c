"""ZeRO-3 per-layer gathers: zero_gather_unit and the prefetching schedule, against the
oracle.

rkmt.cn/news/44736 "Deepspeed ZeRO-3": each layer's parameters are gathered from the
ranks that hold them before the layer's forward pass, and again before its backward
pass.  Here the shards are those the CUDA step wrote for stage 3, and every gathered
unit must equal the oracle's fully gathered parameters (oracle.run_steps, which gathers
unit by unit from its own shards) over the unit's range, bit for bit, for aligned and
unaligned unit starts.  Under the prefetching schedule each layer's "compute" (a
deliberate delay, then a copy of the gathered buffer to the unit's place in an output
buffer) must see its own unit's parameters: a slot overwritten before its layer
finished would show up as a mismatch against the oracle.
"""
import pytest

from seeded_inputs.workloads import reduced_workloads
import zero_sharded_optimizer_ring_b200 as zs
from zero_sharded_optimizer_ring_b200.schedule import GatherWidth, Zero3Prefetch, zero3_pass
import support as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _workload(aligned=True):
    wl = reduced_workloads()["llama3b_n8_zero3"]
    if not aligned:     # a 3-element first tensor moves every later unit start off the 8-grid
        wl = wl.with_(name=wl.name + "_unaligned", tensors=(3,) + tuple(wl.tensors)[1:])
    return wl


def _stepped_shards(wl):
    """Run the CUDA step for the workload's steps; returns the layout, the stage-3 shard
    buffer it wrote, and the oracle's result on the same seeded inputs."""
    ref, _ = S.oracle_run(wl)
    lay = zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align,
                    list(wl.units)).to_device()
    P = lay.padded
    g, master, m, v = S.device_inputs(wl, P)
    p16_shard = torch.zeros(P, dtype=torch.int16, device="cuda")
    p16_full = torch.zeros(P, dtype=torch.int16, device="cuda")
    for t in range(1, wl.steps + 1):
        zs.step(lay, g, master, m, v, p16_shard, p16_full,
                zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale, t))
    zs.get_error(lay)
    torch.cuda.synchronize()
    S.assert_bits_equal(S.to_np(p16_shard), ref.p16_shard, "p16_shard")
    return lay, p16_shard, ref


@pytest.mark.parametrize("gather_ctas", [0, 1, 3, 16])
@pytest.mark.parametrize("aligned", [True, False])
def test_gather_unit_matches_oracle(aligned, gather_ctas):
    wl = _workload(aligned)
    lay, shard, ref = _stepped_shards(wl)
    lay.set_gather_ctas(gather_ctas)            # the grid is the caller's choice; results are not
    _, _, _, u = lay.tables()
    assert aligned == all(lo % 8 == 0 for lo, _ in u)
    for k, (lo, hi) in enumerate(u):
        dst = torch.full((hi - lo + 16,), 7, dtype=torch.int16, device="cuda")
        zs.gather_unit(lay, k, shard, dst)
        torch.cuda.synchronize()
        got = S.to_np(dst)
        S.assert_bits_equal(got[:hi - lo], ref.p16_full[lo:hi], f"unit {k}")
        assert (got[hi - lo:] == 7).all(), f"unit {k}: write past the unit"


@pytest.mark.parametrize("gather_ctas", [1, 5, 148])
@pytest.mark.parametrize("aligned", [True, False])
def test_capped_allgather_matches_oracle(aligned, gather_ctas):
    """zero_allgather (whole buffer and unit by unit, unaligned unit edges included) on a
    capped grid writes exactly the oracle's gathered parameters and nothing else."""
    wl = _workload(aligned)
    lay, shard, ref = _stepped_shards(wl)
    lay.set_gather_ctas(gather_ctas)
    _, _, _, u = lay.tables()
    full = torch.full((lay.padded + 64,), 7, dtype=torch.int16, device="cuda")
    zs.allgather(lay, -1, shard, full[:lay.padded])
    torch.cuda.synchronize()
    S.assert_bits_equal(S.to_np(full)[:lay.padded], ref.p16_full, "whole buffer")
    assert (S.to_np(full)[lay.padded:] == 7).all()
    full.fill_(7)
    for k in range(lay.n_units):
        zs.allgather(lay, k, shard, full[:lay.padded])
    torch.cuda.synchronize()
    S.assert_bits_equal(S.to_np(full)[:lay.padded], ref.p16_full, "unit by unit")
    assert (S.to_np(full)[lay.padded:] == 7).all()


@pytest.mark.parametrize("gather_ctas", [1, 7])
def test_capped_gather_of_a_large_unit_matches_oracle(gather_ctas):
    """One 3,000,017-element unit (ZeRO-3 over the flat list): 123 bulk-copy chunks, many
    per CTA, so every stage of each CTA's shared-memory ring is reloaded many times."""
    wl = reduced_workloads()["flat1p3b_n4_zero1"].with_(stage=3, steps=2)
    lay, shard, ref = _stepped_shards(wl)
    lay.set_gather_ctas(gather_ctas)
    dst = torch.full((lay.padded + 24,), 7, dtype=torch.int16, device="cuda")
    zs.gather_unit(lay, 0, shard, dst)
    full = torch.full((lay.padded + 24,), 7, dtype=torch.int16, device="cuda")
    zs.allgather(lay, 0, shard, full[:lay.padded])
    zs.get_error(lay)
    torch.cuda.synchronize()
    for name, buf in (("gather_unit", dst), ("allgather", full)):
        got = S.to_np(buf)
        S.assert_bits_equal(got[:lay.padded], ref.p16_full, name)
        assert (got[lay.padded:] == 7).all(), f"{name}: write past the unit"


@pytest.mark.parametrize("gather_ctas", [0, None, "width"])
@pytest.mark.parametrize("n_slots", [1, 2, 3])
@pytest.mark.parametrize("backward", [False, True])
def test_prefetch_schedule_gives_each_layer_its_parameters(n_slots, backward, gather_ctas):
    """gather_ctas 0: the gathers' default grid; None: the schedule's own setting;
    "width": a GatherWidth, over three passes (a warm-up, then two timed ones)."""
    wl = _workload()
    lay, shard, ref = _stepped_shards(wl)
    _, _, _, u = lay.tables()
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
    width = GatherWidth() if gather_ctas == "width" else None
    kw = {} if gather_ctas is None else {"gather_ctas": width if width else gather_ctas}
    for _ in range(3 if width else 1):
        out.zero_()
        torch.cuda.synchronize()
        zero3_pass(lay, shard, slots, order, compute, gs, cs, **kw)
        torch.cuda.synchronize()
        assert lay.gather_ctas == 0                 # the layout's setting is restored
        S.assert_bits_equal(S.to_np(out), ref.p16_full, "layers as the compute saw them")
    if width:
        assert sum(width.count) == 1                # the first pass untimed, the third read the second


@pytest.mark.parametrize("n_slots", [2, 3])
def test_passes_enqueued_back_to_back_reuse_slots_safely(n_slots):
    """Zero3Prefetch: a forward, a backward and a forward pass enqueued with no host
    synchronisation between them.  The slots are reused across passes (with three slots
    the backward pass gathers unit 4 into the slot the forward pass's unit 3 is still
    being computed from), so each pass's first gathers must wait for the previous pass's
    layers; every layer of every pass must see exactly its own parameters."""
    wl = _workload()
    lay, shard, ref = _stepped_shards(wl)
    _, _, _, u = lay.tables()
    width = int(max(hi - lo for lo, hi in u))
    slots = [torch.zeros(width, dtype=torch.int16, device="cuda") for _ in range(n_slots)]
    outs = [torch.zeros(lay.padded, dtype=torch.int16, device="cuda") for _ in range(3)]

    def layer(out):
        def compute(unit, buf):
            torch.cuda._sleep(400_000)              # a slow layer: a gather into its slot would overtake it
            lo, hi = int(u[unit][0]), int(u[unit][1])
            out[lo:hi].copy_(buf[:hi - lo])
        return compute

    gs, cs = torch.cuda.Stream(), torch.cuda.Stream()
    pf = Zero3Prefetch(lay, shard, slots, gs, cs, candidates=(2, 16), trials=1)
    torch.cuda.synchronize()
    pf.forward(layer(outs[0]))
    pf.backward(layer(outs[1]))
    pf.forward(layer(outs[2]))
    torch.cuda.synchronize()
    assert lay.gather_ctas == 0
    for k, out in enumerate(outs):
        S.assert_bits_equal(S.to_np(out), ref.p16_full, f"pass {k}: layers as the compute saw them")
