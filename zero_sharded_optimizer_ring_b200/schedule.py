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
# as a few persistent CTAs (zero_set_gather_ctas; 16 unless a GatherWidth tunes it per
# kind of pass) instead of a grid that floods every SM between GEMM waves, and the
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


class GatherWidth:
    """The capped gathers' grid for one kind of pass, chosen by measurement (keep one per
    kind: a forward and a backward pass compute for different times per layer and share
    the GPU differently with their gathers).  Pass it to zero3_pass as gather_ctas.  The
    first pass is a warm-up (a process's first pass also pays one-time start-up costs);
    the next ones try each candidate width in turn, `trials` passes each, rounds
    alternating direction so that a steady drift of the clocks adds the same to every
    candidate; each pass is timed whole (its first event to its last layer's end)
    and read at the start of a later pass once finished, never waiting.  Then the width
    with the lowest mean pass time is kept.  The pass time is the objective because
    neither the waits nor the gathers' speed alone is: a narrower grid that keeps pace
    still runs longer beside more GEMM waves, and a wider one takes SMs from them."""

    def __init__(self, candidates=(14, 16, 18, 20), trials=3):
        candidates = tuple(int(c) for c in candidates)
        if not candidates or min(candidates) < 1 or trials < 1:
            raise ValueError("need at least one candidate width >= 1 and trials >= 1")
        self.candidates, self.trials = candidates, int(trials)
        self.sum_ms = [0.0] * len(candidates)
        self.count = [0] * len(candidates)
        self.chosen = None          # index into candidates, once every one is timed
        self._pending = None        # (candidate index, marks, pass start) not yet read
        self._timing = None         # candidate index of the pass being enqueued
        self._warm = False          # the untimed first pass has been enqueued

    @property
    def ctas(self):
        """The width the next pass uses."""
        return self.candidates[self._next()]

    def means(self):
        """Mean pass time (ms) per candidate so far (None where untimed)."""
        return [s / n if n else None for s, n in zip(self.sum_ms, self.count)]

    def observe(self):
        """Read the pending pass if its events have completed."""
        if self._pending is None:
            return
        i, marks, start = self._pending
        if marks and not marks[-1][2].query():
            return                  # still running: read it before a later pass
        self._pending = None
        if marks:
            self.sum_ms[i] += start.elapsed_time(marks[-1][2])
            self.count[i] += 1
        if self.chosen is None and min(self.count) >= self.trials:
            means = self.means()
            self.chosen = min(range(len(means)), key=lambda k: means[k])

    def begin_pass(self):
        """Read the last pass if it has finished; the width the starting pass uses."""
        self.observe()
        self._timing = self._next() if self.chosen is None and self._warm else None
        self._warm = True
        return self.candidates[self._next()]

    def end_pass(self, marks, start):
        """Leave the pass just enqueued (its zero3_pass events and start event) to be
        read at the start of a later one."""
        if self._timing is not None:
            self._pending = (self._timing, marks, start)

    def _next(self):
        if self.chosen is not None:
            return self.chosen
        K = len(self.candidates)
        lo = min(self.count)
        order = range(K) if lo % 2 == 0 else range(K - 1, -1, -1)
        return next(k for k in order if self.count[k] == lo)


class Zero3Prefetch:
    """ZeRO-3's gathers for a training loop: the slot ring, the two streams and one
    GatherWidth per kind of pass, kept across steps.  forward() and backward() run
    zero3_pass over the units in ascending and descending order with that kind's width;
    the widths settle on their own over the first steps (candidates x trials + 1 passes
    of each kind).  `gather` as for zero3_pass (one GPU per rank: RankStep.prefetch)."""

    def __init__(self, layout, p16_shard, slots, gather_stream, compute_stream, candidates=(14, 16, 18, 20),
                 trials=3, matmul_sm_carveout=MATMUL_SM_CARVEOUT, blas=MATMUL_BLAS, gather=None):
        self.layout, self.p16_shard, self.slots = layout, p16_shard, list(slots)
        self.gather_stream, self.compute_stream = gather_stream, compute_stream
        self.widths = {"forward": GatherWidth(candidates, trials), "backward": GatherWidth(candidates, trials)}
        self.matmul_sm_carveout, self.blas, self.gather = matmul_sm_carveout, blas, gather

    def _run(self, kind, units, compute):
        return zero3_pass(self.layout, self.p16_shard, self.slots, units, compute, self.gather_stream,
                          self.compute_stream, gather_ctas=self.widths[kind],
                          matmul_sm_carveout=self.matmul_sm_carveout, blas=self.blas, gather=self.gather)

    def forward(self, compute, units=None):
        """The forward pass: units ascending (default: all of the layout's)."""
        return self._run("forward", list(range(self.layout.n_units)) if units is None else units, compute)

    def backward(self, compute, units=None):
        """The backward pass: units descending (default: all of the layout's)."""
        return self._run("backward", list(range(self.layout.n_units))[::-1] if units is None else units, compute)


def zero3_pass(layout, p16_shard, slots, units, compute, gather_stream, compute_stream,
               gather_ctas=GATHER_CTAS, matmul_sm_carveout=MATMUL_SM_CARVEOUT, blas=MATMUL_BLAS, gather=None):
    """Run one pass over `units` (a forward pass: ascending; a backward pass: descending).

    Unit units[j] is gathered into slots[j % len(slots)] on gather_stream, once the slot's
    previous occupant units[j - len(slots)] has been computed; compute(unit, buffer) is
    then called with compute_stream current and must enqueue the layer's work there.
    During the pass the gathers run on gather_ctas persistent CTAs (an int; a GatherWidth,
    whose current width is used and which then reads this pass; None: the layout's
    setting), except the first len(slots), which are issued before any layer has computed
    and so take the whole GPU; torch's matmuls run with the SM-count target
    matmul_sm_carveout below the SM count and prefer `blas` (None: unchanged); every
    setting is restored afterwards.  The first gathers wait for the work already on
    compute_stream (an earlier pass's layers may still read the slots).  gather(unit, dst,
    stream) enqueues a unit's parameters into dst (default: zero_gather_unit from
    p16_shard; with one GPU per rank, RankStep.gather_unit, which reads every owner's
    shard and honours the same gather width).  Returns the list
    of (gather started, gathered, computed) torch.cuda.Event triples, one per unit (timing
    events: layer_breakdown reads them)."""
    import torch
    n = len(slots)
    marks = []
    if gather is None:
        def gather(unit, dst, stream):
            gather_unit(layout, unit, p16_shard, dst, stream=stream)
    width = gather_ctas if isinstance(gather_ctas, GatherWidth) else None
    if width is not None:
        gather_ctas = width.begin_pass()
    saved_ctas = layout.gather_ctas
    pass_start = torch.cuda.Event(enable_timing=True)
    pass_start.record(compute_stream)
    gather_stream.wait_event(pass_start)
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
                gather(u, slots[j % n], gather_stream)
                gathered.record(gather_stream)
                compute_stream.wait_event(gathered)
                with torch.cuda.stream(compute_stream):
                    compute(u, slots[j % n])
                computed.record(compute_stream)
                marks.append((started, gathered, computed))
    finally:
        layout.set_gather_ctas(saved_ctas)
    if width is not None:
        width.end_pass(marks, pass_start)
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
