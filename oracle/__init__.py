"""CPU oracle of the data-parallel optimizer step (DDP and ZeRO-1/2/3).
TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and bench.py's CPU-baseline /
reference arm use it; the CUDA library never does, and shares no code with it.

It computes, literally and slowly, what the pages describe for N data-parallel ranks
holding fp16 gradients of psi parameters:
  1. per bucket, a ring scatter-reduce: chunk k starts at rank k and is passed around
     the ring, each rank adding its own fp32-converted gradient (en.pswp.cn/web/84187
     "DDP", the three-GPU Ring-AllReduce walk-through);
  2. per shard, the update: scale the sum by 1/(N*loss_scale), AdamW on the fp32 first
     and second moments and fp32 master weights, fp16 parameter write (rkmt.cn/news/44736
     "Deepspeed ZeRO-1", update step);
  3. a ring all-gather of the fp16 shards into the full parameter buffer (same page,
     broadcast step; wangyh.co PaperReading:DeepSpeed section 2.5, all-gather = the
     concatenation of every rank's partition), per gather unit (layer) for ZeRO-3
     (rkmt.cn/news/44736 "Deepspeed ZeRO-3": parameters broadcast layer by layer).
DDP (stage 0) instead all-gathers the reduced gradients and every rank updates the
full vector (rkmt.cn/news/44736 "DDP"; wangyh.co section 1.1).

Parity pins for every function live in tests/test_oracle_*.py.
"""
import ctypes
from dataclasses import dataclass

import numpy as np

from . import build as _build
from .layout import OracleLayout, OracleCounters, make_layout, counters  # noqa: F401

_LIB = None
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_dbl = ctypes.c_double


def lib():
    global _LIB
    if _LIB is None:
        _build.build()
        _LIB = configure(ctypes.CDLL(_build.LIB))
    return _LIB


def configure(L):
    """Declare the C functions' signatures on a loaded oracle library."""
    L.oracle_half_to_float.argtypes = [ctypes.c_uint16]
    L.oracle_half_to_float.restype = ctypes.c_float
    L.oracle_float_to_half.argtypes = [ctypes.c_float]
    L.oracle_float_to_half.restype = ctypes.c_uint16
    L.oracle_halfs_to_floats.argtypes = [_vp, _vp, _i64]
    L.oracle_floats_to_halfs.argtypes = [_vp, _vp, _i64]
    L.oracle_double_to_half.argtypes = [_dbl]
    L.oracle_double_to_half.restype = ctypes.c_uint16
    L.oracle_ring_reduce_scatter.argtypes = [_vp, _i32, _i64, _i64, _i64, _i64, _i32, _i32,
                                             _vp, _vp, _vp, _vp, _vp]
    L.oracle_ring_reduce_scatter.restype = _i64
    L.oracle_ring_allgather.argtypes = [_vp, _i32, _i32, _i64, _i64, _i64, _i64, _vp, _vp, _vp]
    L.oracle_ring_allgather.restype = _i64
    L.oracle_adamw_scalars.argtypes = [_vp, _i32, _dbl, _dbl, _dbl, _dbl, _dbl, _dbl, _i64]
    L.oracle_adamw.argtypes = [_i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]
    L.oracle_count_nonfinite.argtypes = [_vp, _i64, _i64]
    L.oracle_count_nonfinite.restype = _i64
    L.oracle_sampled.argtypes = [_i64, _i32, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp]
    return L


def _p(a):
    return None if a is None else a.ctypes.data_as(_vp)


def _need(a, dtype):
    assert a.dtype == dtype and a.flags["C_CONTIGUOUS"], (a.dtype, dtype)
    return a


# ---------------------------------------------------------------- primitives

def half_to_float(bits):
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float32)
    lib().oracle_halfs_to_floats(_p(bits), _p(out), bits.size)
    return out


def float_to_half(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().oracle_floats_to_halfs(_p(x), _p(out), x.size)
    return out


@dataclass(frozen=True)
class Hyper:
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.01
    loss_scale: float = 1.0


def adamw_scalars(n_ranks, hp, t):
    s = np.zeros(9, dtype=np.float32)
    lib().oracle_adamw_scalars(_p(s), n_ranks, hp.loss_scale, hp.lr, hp.beta1, hp.beta2,
                               hp.eps, hp.weight_decay, t)
    return s


def ring_reduce_scatter(grads, shard, blo, bhi, hops=None, reduced=None, sent=None, recv=None,
                        want_log=False, wire16=False):
    """Scatter-reduce of bucket [blo, bhi).  grads: uint16 [N, rank_stride] fp16 bits.
    wire16: partials travel as fp16 (each hop's sum rounded to fp16).
    Returns (work [N, bhi-blo] running partials per rank, log [n, 4] or None)."""
    _need(grads, np.uint16)
    N, stride = grads.shape
    hops = N - 1 if hops is None else hops
    work = np.zeros((N, bhi - blo), dtype=np.float32)
    log = np.zeros((max(1, N * hops), 4), dtype=np.int64) if want_log else None
    n = lib().oracle_ring_reduce_scatter(_p(grads), N, stride, shard, blo, bhi, hops, int(wire16), _p(work),
                                         _p(reduced), _p(log), _p(sent), _p(recv))
    return work, (log[:n] if want_log else None)


def ring_allgather(rep, shard, lo, hi, sent=None, recv=None, want_log=False):
    """All-gather of [lo, hi) across the replicas rep [N, stride] (any element type)."""
    assert rep.flags["C_CONTIGUOUS"]
    N, stride = rep.shape
    log = np.zeros((max(1, N * (N - 1)), 4), dtype=np.int64) if want_log else None
    n = lib().oracle_ring_allgather(_p(rep), rep.itemsize, N, stride, shard, lo, hi,
                                    _p(log), _p(sent), _p(recv))
    return log[:n] if want_log else None


def adamw(lo, hi, reduced, master, m, v, p16, scalars):
    for a in (reduced, master, m, v, scalars):
        _need(a, np.float32)
    _need(p16, np.uint16)
    lib().oracle_adamw(lo, hi, _p(reduced), _p(master), _p(m), _p(v), _p(p16), _p(scalars))


def count_nonfinite(reduced, lo, hi):
    return int(lib().oracle_count_nonfinite(_p(_need(reduced, np.float32)), lo, hi))


def double_to_half(x):
    return int(lib().oracle_double_to_half(float(x)))


def sampled(g, shard_of, steps, scalars, master, m, v, wire16=False):
    """Per-element path: g uint16 [n, N]; shard_of int64 [n]; scalars float32 [steps, 9];
    master/m/v float32 [n] (updated in place).  Returns (reduced, p16)."""
    g = np.ascontiguousarray(g, dtype=np.uint16)
    n, N = g.shape
    shard_of = np.ascontiguousarray(shard_of, dtype=np.int64)
    scalars = np.ascontiguousarray(scalars, dtype=np.float32)
    for a in (master, m, v):
        _need(a, np.float32)
    reduced = np.zeros(n, dtype=np.float32)
    p16 = np.zeros(n, dtype=np.uint16)
    lib().oracle_sampled(n, N, _p(g), _p(shard_of), int(wire16), steps, _p(scalars), _p(reduced),
                         _p(master), _p(m), _p(v), _p(p16))
    return reduced, p16


# ---------------------------------------------------------------- whole steps

@dataclass
class StepResult:
    master: np.ndarray        # fp32 [P]
    m: np.ndarray
    v: np.ndarray
    p16_full: np.ndarray      # fp16 bits [P]: full parameter buffer after the gather
    p16_shard: np.ndarray     # fp16 bits [P]: concatenated shards (written by the update)
    reduced: np.ndarray       # fp32 [P]: ring sums of the last step (before scaling)
    nonfinite: np.ndarray     # int64 [n_buckets]: non-finite ring sums, last step
    sent: np.ndarray          # int64 [N]: elements sent per rank, all steps (literal)
    recv: np.ndarray
    replicas_identical: bool  # with replicas=True: every rank ended with the same values


def run_steps(lay, stage, grads, master, m, v, hp, steps, replicas=False, wire16=False, first_step=1):
    """Run `steps` optimizer steps of ZeRO stage `stage` (0 = DDP) on the oracle.

    grads: uint16 [N, rank_stride >= P] fp16 bits (the same at every step);
    master, m, v: float32 [P] initial state (copied, not modified).
    replicas=True keeps every rank's copy of the replicated buffers and runs the
    all-gathers hop by hop (tiny cases); otherwise one copy stands for all ranks and
    the gathers are the plain copies they reduce to.
    """
    N, S, P = lay.n_ranks, lay.shard, lay.padded
    assert grads.shape[0] == N and grads.shape[1] >= P
    master, m, v = (np.array(x, dtype=np.float32, copy=True) for x in (master, m, v))
    sent = np.zeros(N, dtype=np.int64)
    recv = np.zeros(N, dtype=np.int64)
    reps = N if replicas else 1
    if stage == 0:   # DDP keeps the full optimizer state on every rank
        st = [[x.copy() for x in (master, m, v)] for _ in range(reps)]
    p16_full = np.zeros((reps, P), dtype=np.uint16)
    p16_shard = np.zeros(P, dtype=np.uint16)
    reduced = np.zeros(P, dtype=np.float32)
    nonfinite = np.zeros(len(lay.buckets), dtype=np.int64)

    for t in range(first_step, first_step + steps):
        sc = adamw_scalars(N, hp, t)
        reduced[:] = 0
        for b, (lo, hi) in enumerate(lay.buckets):
            ring_reduce_scatter(grads, S, lo, hi, reduced=reduced, sent=sent, recv=recv, wire16=wire16)
            nonfinite[b] = count_nonfinite(reduced, lo, hi)

        if stage == 0:
            # all-reduce = scatter-reduce + all-gather of the sums; every rank updates all
            red = np.tile(reduced, (reps, 1))
            if replicas:
                for lo, hi in lay.buckets:
                    ring_allgather(red, S, lo, hi, sent=sent, recv=recv)
            for r in range(reps):
                mr, mm, vv = st[r]
                adamw(0, P, np.ascontiguousarray(red[r]), mr, mm, vv, p16_full[r], sc)
            master, m, v = st[0]
        else:
            for k in range(N):
                adamw(k * S, (k + 1) * S, reduced, master, m, v, p16_shard, sc)
            holder_views = p16_full if stage != 3 else None
            if stage in (1, 2):
                # the rank where shard k's reduction completed holds its new fp16 values,
                # then broadcasts them around the ring
                for k in range(N):
                    h = (k - 1) % N if replicas else 0
                    p16_full[h, k * S:(k + 1) * S] = p16_shard[k * S:(k + 1) * S]
                if replicas:
                    ring_allgather(holder_views, S, 0, P, sent=sent, recv=recv)
            else:
                # ZeRO-3: the full parameters exist only while a layer is gathered
                p16_full[:] = 0
                for ulo, uhi in lay.units:
                    for k in range(N):
                        a, z = max(ulo, k * S), min(uhi, (k + 1) * S)
                        if z > a:
                            h = (k - 1) % N if replicas else 0
                            p16_full[h, a:z] = p16_shard[a:z]
                    if replicas:
                        ring_allgather(p16_full, S, ulo, uhi, sent=sent, recv=recv)

    same = True
    if replicas:
        same = all(np.array_equal(p16_full[0], p16_full[r]) for r in range(N))
        if stage == 0:
            same = same and all(np.array_equal(st[0][j], st[r][j]) for r in range(N) for j in range(3))
    if stage == 0:
        p16_shard = p16_full[0].copy()
    return StepResult(master, m, v, p16_full[0].copy(), p16_shard, reduced.copy(), nonfinite,
                      sent, recv, same)


# ---------------------------------------------------------------- dynamic loss scaling

@dataclass
class LossScaler:
    """Dynamic loss scaling (mixed-precision training practice; the pages do not spell it
    out): gradients arrive multiplied by `scale`.  A step whose reduced gradients hold a
    non-finite value is skipped (no state changes) and the scale is divided by `factor`
    (not below `min_scale`); after `window` consecutive applied steps it is multiplied by
    `factor`.  `step` counts applied AdamW steps (the next applied step uses step + 1)."""
    scale: float
    factor: float = 2.0
    window: int = 1000
    min_scale: float = 1.0
    clean_steps: int = 0
    step: int = 0
    skipped: int = 0

    def update(self, overflow):
        if overflow:
            self.scale = max(self.scale / self.factor, self.min_scale)
            self.clean_steps = 0
            self.skipped += 1
        else:
            self.step += 1
            self.clean_steps += 1
            if self.clean_steps == self.window:
                self.scale *= self.factor
                self.clean_steps = 0


def run_steps_dynamic(lay, stage, grads_at, master, m, v, hp, steps, scaler, wire16=False):
    """`steps` training steps under dynamic loss scaling.  grads_at(scale, i) gives step i's
    fp16 gradients [N, >= P] produced at loss scale `scale`.  Each step reduces every
    bucket (ring order, fp32 or fp16 wire), and applies the update with the scale the
    gradients carry only if no reduced value is non-finite.  Returns (result of the last
    applied step or None, trace of (scale used, overflow, AdamW step or 0) per step)."""
    N, S = lay.n_ranks, lay.shard
    state = [np.array(x, dtype=np.float32, copy=True) for x in (master, m, v)]
    last = None
    trace = []
    for i in range(steps):
        g = grads_at(scaler.scale, i)
        reduced = np.zeros(lay.padded, dtype=np.float32)
        bad = 0
        for lo, hi in lay.buckets:
            ring_reduce_scatter(g, S, lo, hi, reduced=reduced, wire16=wire16)
            bad += count_nonfinite(reduced, lo, hi)
        used = scaler.scale
        if bad == 0:
            h = Hyper(hp.lr, hp.beta1, hp.beta2, hp.eps, hp.weight_decay, used)
            last = run_steps(lay, stage, g, *state, h, 1, wire16=wire16, first_step=scaler.step + 1)
            state = [last.master, last.m, last.v]
        scaler.update(bad > 0)
        trace.append((used, bad > 0, scaler.step if bad == 0 else 0))
    return last, trace
