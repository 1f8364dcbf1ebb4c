"""ZeRO-3 layer-by-layer parameter gathering with prefetch (host-side scheduling only).

rkmt.cn/news/44736 "Deepspeed ZeRO-3": before a layer's forward, and again before its
backward, its parameters are gathered from the ranks that hold them, and released once
the layer is done; the forward and backward gathers plus the gradient reduce-scatter
make the 3 psi per GPU of ZeRO-3.  Here each unit (layer) is gathered with
zero_gather_unit into one slot of a small ring of unit-sized buffers, so only
len(slots) layers are materialised at a time; with two or more slots the gather of the
next layer runs on its own stream while the current layer computes.  Every gather is a
library kernel; the schedule is CUDA stream waits and events.
"""
from . import gather_unit


def zero3_pass(layout, p16_shard, slots, units, compute, gather_stream, compute_stream):
    """Run one pass over `units` (a forward pass: ascending; a backward pass: descending).

    Unit units[j] is gathered into slots[j % len(slots)] on gather_stream, once the slot's
    previous occupant units[j - len(slots)] has been computed; compute(unit, buffer) is
    then called with compute_stream current and must enqueue the layer's work there.
    Returns the list of (gather started, gathered, computed) torch.cuda.Event triples,
    one per unit (timing events: layer_breakdown reads them)."""
    import torch
    n = len(slots)
    marks = []
    for j, u in enumerate(units):
        started, gathered, computed = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        if j >= n:
            gather_stream.wait_event(marks[j - n][2])
        started.record(gather_stream)
        gather_unit(layout, u, p16_shard, slots[j % n], stream=gather_stream)
        gathered.record(gather_stream)
        compute_stream.wait_event(gathered)
        with torch.cuda.stream(compute_stream):
            compute(u, slots[j % n])
        computed.record(compute_stream)
        marks.append((started, gathered, computed))
    return marks


def layer_breakdown(marks, pass_start):
    """Where one pass's time went, from the events zero3_pass recorded (after they have
    completed): per layer, the gather's own duration, the time the compute stream sat
    waiting for that gather (the exposed gather), and the layer's compute time.  Returns
    a dict of per-layer lists (ms) and their sums."""
    gather, wait, compute = [], [], []
    prev = pass_start
    for started, gathered, computed in marks:
        g = started.elapsed_time(gathered)
        w = max(0.0, prev.elapsed_time(gathered))          # compute ready before its parameters
        total = prev.elapsed_time(computed)
        gather.append(g)
        wait.append(w)
        compute.append(total - w)
        prev = computed
    return {"gather_ms": gather, "wait_ms": wait, "compute_ms": compute,
            "sum_gather_ms": sum(gather), "sum_wait_ms": sum(wait), "sum_compute_ms": sum(compute)}
