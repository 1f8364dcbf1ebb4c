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


# How the gathers share the GPU with the layers' GEMMs during a pass (measured on the
# Llama-shaped list, 2048 tokens, two slots): the gathers issued once layers compute run
# as 16 persistent CTAs
# (zero_set_gather_ctas) instead of a grid that floods every SM between GEMM waves, and the
# matmuls run with cuBLAS's SM-count target 16 below the SM count on the cuBLASLt path
# (torch's matmul carveout).  The target is a hint to the GEMM kernel choice rather than a
# cap on the SMs a GEMM occupies; with it the layer GEMMs alone are no slower, and beside
# the capped gathers both passes expose less gather time than without prefetch.
GATHER_CTAS = 16
MATMUL_SM_CARVEOUT = 16
MATMUL_BLAS = "cublaslt"


class _MatmulShare:
    """Within the block, torch's matmuls run with cuBLAS's SM-count target `carveout` SMs
    below the SM count and prefer `blas` (either None: unchanged); both restored on exit."""

    def __init__(self, carveout, blas):
        self.carveout, self.blas = carveout, blas

    def __enter__(self):
        import torch
        self.saved_carveout = self.saved_blas = None
        if self.carveout is not None and hasattr(torch._C, "_set_sm_carveout_experimental"):
            self.saved_carveout = (torch._C._get_sm_carveout_experimental(),)
            torch._C._set_sm_carveout_experimental(self.carveout or None)
        if self.blas is not None:
            self.saved_blas = (torch.backends.cuda.preferred_blas_library(),)
            torch.backends.cuda.preferred_blas_library(self.blas)
        return self

    def __exit__(self, *exc):
        import torch
        if self.saved_carveout is not None:
            torch._C._set_sm_carveout_experimental(self.saved_carveout[0])
        if self.saved_blas is not None:
            torch.backends.cuda.preferred_blas_library(self.saved_blas[0])


def zero3_pass(layout, p16_shard, slots, units, compute, gather_stream, compute_stream,
               gather_ctas=GATHER_CTAS, matmul_sm_carveout=MATMUL_SM_CARVEOUT, blas=MATMUL_BLAS):
    """Run one pass over `units` (a forward pass: ascending; a backward pass: descending).

    Unit units[j] is gathered into slots[j % len(slots)] on gather_stream, once the slot's
    previous occupant units[j - len(slots)] has been computed; compute(unit, buffer) is
    then called with compute_stream current and must enqueue the layer's work there.
    During the pass the gathers run on gather_ctas persistent CTAs (None: the layout's
    setting), except the first len(slots), which are issued before any layer has computed
    and so take the whole GPU; torch's matmuls run with the SM-count target
    matmul_sm_carveout below the SM count and prefer `blas` (None: unchanged); every
    setting is restored afterwards.  Returns the list of (gather started, gathered,
    computed) torch.cuda.Event triples, one per unit (timing events: layer_breakdown reads
    them)."""
    import torch
    n = len(slots)
    marks = []
    saved_ctas = layout.gather_ctas
    try:
        with _MatmulShare(matmul_sm_carveout, blas):
            for j, u in enumerate(units):
                started, gathered, computed = (torch.cuda.Event(enable_timing=True) for _ in range(3))
                if j >= n:
                    gather_stream.wait_event(marks[j - n][2])
                if gather_ctas is not None:
                    # the first n gathers have no layer compute to share the GPU with
                    layout.set_gather_ctas(0 if j < n else gather_ctas)
                started.record(gather_stream)
                gather_unit(layout, u, p16_shard, slots[j % n], stream=gather_stream)
                gathered.record(gather_stream)
                compute_stream.wait_event(gathered)
                with torch.cuda.stream(compute_stream):
                    compute(u, slots[j % n])
                computed.record(compute_stream)
                marks.append((started, gathered, computed))
    finally:
        layout.set_gather_ctas(saved_ctas)
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
