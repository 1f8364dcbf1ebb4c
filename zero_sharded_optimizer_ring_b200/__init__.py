"""Sharded data-parallel optimizer step (DDP, ZeRO-1/2/3) for one B200.

A thin binding over the C ABI of include/zero.h: it turns torch tensors into device
pointers and a CUDA stream handle, and status codes into exceptions.  Every step of
the computation runs in the library's CUDA kernels (libzero_b200.so).

    lay = Layout(tensor_sizes, n_ranks=8, stage=2, bucket_elems=25_000_000)
    lay.to_device()
    step(lay, grads, master, m, v, None, p16_full, AdamW(lr=1e-3, loss_scale=1024, step=t))
"""
import ctypes
from dataclasses import dataclass

import numpy as np

from . import _abi

__all__ = ["ZeroError", "Layout", "AdamW", "reduce_scatter", "adamw_shard_step", "allgather", "gather_unit", "gather_unit_ranks",
           "step", "step_scalars", "step_device_scalars", "step_bucket", "step_overlapped", "step_dynamic", "step_dynamic_commit", "LossScaler", "step_host",
           "step_noalloc", "step_ranks", "step_shard", "step_shard_commit", "copy_shard", "ipc_handle", "ipc_open", "ipc_close",
           "get_error", "IMPL_AUTO", "IMPL_REGISTER", "IMPL_BULK"]

IMPL_AUTO, IMPL_REGISTER, IMPL_BULK = 0, 1, 2


class ZeroError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        msg = _abi.lib().zero_status_string(status).decode()
        super().__init__(f"{what}: {_abi.STATUS_NAMES.get(status, status)} ({msg})")


def _check(status, what):
    if status != _abi.ZERO_OK:
        raise ZeroError(status, what)


def _ptr(t):
    """Device (or host) address of a torch tensor, an int address, or None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


@dataclass
class AdamW:
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.01
    loss_scale: float = 1.0
    step: int = 1

    def c(self):
        return _abi.AdamWHparams(self.lr, self.beta1, self.beta2, self.eps, self.weight_decay,
                                 self.loss_scale, self.step)


class Layout:
    """Flat buffer, shards, buckets, segments and gather units (zero_layout_create)."""

    def __init__(self, tensors, n_ranks, stage, bucket_elems=0, pad_align=128, units=(), wire_fp16=False):
        lib = _abi.lib()
        self._numel = (ctypes.c_int64 * max(1, len(tensors)))(*[int(x) for x in tensors])
        self._units = (ctypes.c_int64 * max(1, len(units)))(*[int(x) for x in units])
        desc = _abi.LayoutDesc(int(n_ranks), int(stage), len(tensors), self._numel, int(bucket_elems),
                               int(pad_align), len(units), self._units, int(bool(wire_fp16)))
        h = ctypes.c_void_p()
        _check(lib.zero_layout_create(ctypes.byref(desc), ctypes.byref(h)), "zero_layout_create")
        self._h = h
        self.n_ranks = int(n_ranks)
        self.stage = int(stage)
        self.n_tensors = len(tensors)
        info = _abi.LayoutInfo()
        _check(lib.zero_layout_get_info(self._h, ctypes.byref(info)), "zero_layout_get_info")
        self.psi, self.shard, self.padded = info.psi, info.shard, info.padded
        self.n_buckets, self.n_segments, self.n_units = info.n_buckets, info.n_segments, info.n_units
        self.tile_elems, self.n_tiles = info.tile_elems, info.n_tiles

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            _abi.lib().zero_layout_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def tables(self):
        """Host copies: tensor_off [T], buckets [B,2], segments [S,4], units [U,2]."""
        t = np.zeros(max(1, self.n_tensors), np.int64)
        b = np.zeros((max(1, self.n_buckets), 2), np.int64)
        s = np.zeros((max(1, self.n_segments), 4), np.int64)
        u = np.zeros((max(1, self.n_units), 2), np.int64)
        _check(_abi.lib().zero_layout_get_tables(self._h, t.ctypes.data, b.ctypes.data, s.ctypes.data,
                                                 u.ctypes.data), "zero_layout_get_tables")
        return t[:self.n_tensors], b[:self.n_buckets], s[:self.n_segments], u[:self.n_units]

    def counters(self):
        c = _abi.Counters()
        _check(_abi.lib().zero_layout_counters(self._h, ctypes.byref(c)), "zero_layout_counters")
        return {f: getattr(c, f) for f, _ in _abi.Counters._fields_}

    def to_device(self, stream=None):
        _check(_abi.lib().zero_layout_to_device(self._h, _stream(stream)), "zero_layout_to_device")
        return self

    def device_segments(self, stream=None):
        out = np.zeros((self.n_segments + 1, 5), np.int64)
        _check(_abi.lib().zero_layout_device_segments(self._h, out.ctypes.data, _stream(stream)),
               "zero_layout_device_segments")
        return out

    def set_impl(self, impl):
        _check(_abi.lib().zero_set_impl(self._h, int(impl)), "zero_set_impl")

    def set_max_ctas(self, max_ctas):
        """At most max_ctas CTAs per fused-step / reduce-scatter launch (0 = all SMs)."""
        _check(_abi.lib().zero_set_max_ctas(self._h, int(max_ctas)), "zero_set_max_ctas")

    def set_gather_ctas(self, max_ctas):
        """All-gather copies as max_ctas persistent CTAs (0 = the default grid of short blocks)."""
        _check(_abi.lib().zero_set_gather_ctas(self._h, int(max_ctas)), "zero_set_gather_ctas")
        self._gather_ctas = int(max_ctas)

    @property
    def gather_ctas(self):
        return getattr(self, "_gather_ctas", 0)

    def overlap_plan(self):
        """(plan, mean ms per plan) the overlapped steps settled on (zero_overlap_plan):
        plan -1 while still timing, 0-3 = grid capped at 1, 2/3, 1/2, 1/3 of the SMs,
        4 = deferred to one launch after the last bucket."""
        plan = ctypes.c_int32()
        means = np.zeros(_abi.OVERLAP_PLANS, np.float32)
        _check(_abi.lib().zero_overlap_plan(self._h, ctypes.byref(plan), means.ctypes.data), "zero_overlap_plan")
        return int(plan.value), [float(x) for x in means]

    def debug_set_wait(self, wait_limit_ns, skip_first_fill=0):
        _check(_abi.lib().zero_debug_set_wait(self._h, int(wait_limit_ns), int(skip_first_fill)),
               "zero_debug_set_wait")


def _stride(grads, layout, rank_stride):
    if rank_stride is not None:
        return int(rank_stride)
    if grads.dim() == 2:
        return int(grads.stride(0))
    return int(layout.padded)


def reduce_scatter(layout, bucket, grads, reduced, nonfinite=None, rank_stride=None, stream=None):
    _check(_abi.lib().zero_reduce_scatter(layout.handle, int(bucket), _ptr(grads),
                                          _stride(grads, layout, rank_stride), _ptr(reduced),
                                          _ptr(nonfinite), _stream(stream)), "zero_reduce_scatter")


def adamw_shard_step(layout, shard, reduced, master, m, v, p16_out, hp, stream=None):
    h = hp.c()
    _check(_abi.lib().zero_adamw_shard_step(layout.handle, int(shard), _ptr(reduced), _ptr(master), _ptr(m),
                                            _ptr(v), _ptr(p16_out), ctypes.byref(h), _stream(stream)),
           "zero_adamw_shard_step")


def allgather(layout, unit, p16_shard, p16_full, stream=None):
    _check(_abi.lib().zero_allgather(layout.handle, int(unit), _ptr(p16_shard), _ptr(p16_full),
                                     _stream(stream)), "zero_allgather")


def gather_unit(layout, unit, p16_shard, dst, stream=None):
    """Unit `unit`'s fp16 parameters, contiguous, into dst (zero_gather_unit)."""
    _check(_abi.lib().zero_gather_unit(layout.handle, int(unit), _ptr(p16_shard), _ptr(dst), _stream(stream)),
           "zero_gather_unit")


def gather_unit_ranks(layout, unit, rank_p16, dst, stream=None):
    """Unit `unit`'s fp16 parameters into dst from the ranks' own shard buffers
    (zero_gather_unit_ranks); rank_p16[k]: tensor or device address of rank k's shard."""
    _check(_abi.lib().zero_gather_unit_ranks(layout.handle, int(unit), _ptr_array(rank_p16), _ptr(dst),
                                             _stream(stream)), "zero_gather_unit_ranks")


def step(layout, grads, master, m, v, p16_shard, p16_full, hp, nonfinite=None, events=None,
         rank_stride=None, stream=None):
    """events: optional dict of torch.cuda.Event (enable_timing) under the keys
    update_begin, update_end, gather_begin, gather_end."""
    h = hp.c()
    ev = None
    if events:
        handles = []
        for k in ("update_begin", "update_end", "gather_begin", "gather_end"):
            e = events.get(k)
            if e is not None and e.cuda_event == 0:
                e.record()          # torch creates the cudaEvent_t on first record
            handles.append(e.cuda_event if e is not None else None)
        ev = _abi.StepEvents(*handles)
    _check(_abi.lib().zero_step(layout.handle, _ptr(grads), _stride(grads, layout, rank_stride), _ptr(master),
                                _ptr(m), _ptr(v), _ptr(p16_shard), _ptr(p16_full), ctypes.byref(h),
                                _ptr(nonfinite), ctypes.byref(ev) if ev is not None else None,
                                _stream(stream)), "zero_step")


def step_scalars(layout, hp):
    """The fp32 scalars of step hp.step (zero_step_scalars_fill) as a float32 numpy array
    of 9, in the order zero_step_device_scalars reads them."""
    out = _abi.StepScalars()
    h = hp.c()
    _check(_abi.lib().zero_step_scalars_fill(layout.handle, ctypes.byref(h), ctypes.byref(out)),
           "zero_step_scalars_fill")
    return np.array([getattr(out, f) for f, _ in _abi.StepScalars._fields_], dtype=np.float32)


def step_device_scalars(layout, grads, master, m, v, p16_shard, p16_full, scalars_dev, nonfinite=None,
                        rank_stride=None, stream=None):
    """zero_step reading its scalars from scalars_dev (a float32 device tensor of 9) when it
    runs (zero_step_device_scalars): capturable once in a CUDA graph and replayed."""
    _check(_abi.lib().zero_step_device_scalars(layout.handle, _ptr(grads), _stride(grads, layout, rank_stride),
                                               _ptr(master), _ptr(m), _ptr(v), _ptr(p16_shard), _ptr(p16_full),
                                               _ptr(scalars_dev), _ptr(nonfinite), _stream(stream)),
           "zero_step_device_scalars")


def step_bucket(layout, bucket, grads, master, m, v, p16_shard, p16_full, hp, nonfinite=None, rank_stride=None,
                stream=None):
    """The fused reduce-scatter + update of one bucket (zero_step_bucket)."""
    h = hp.c()
    _check(_abi.lib().zero_step_bucket(layout.handle, int(bucket), _ptr(grads), _stride(grads, layout, rank_stride),
                                       _ptr(master), _ptr(m), _ptr(v), _ptr(p16_shard), _ptr(p16_full),
                                       ctypes.byref(h), _ptr(nonfinite), _stream(stream)), "zero_step_bucket")


def step_overlapped(layout, ready_events, grads, master, m, v, p16_shard, p16_full, hp, nonfinite=None,
                    rank_stride=None, stream=None, group=None):
    """zero_step with bucket b gated on ready_events[b] (torch.cuda.Event, recorded by the
    producer of bucket b's gradients).  group=None: zero_step_overlapped (small buckets
    coalesced into launches of >= 2^24 elements); an integer: one launch per `group`
    consecutive buckets (zero_step_overlapped_grouped).  Either way the grid cap is the
    layout's (set_max_ctas) or, if none, the library's measured choice."""
    assert len(ready_events) == layout.n_buckets
    handles = (ctypes.c_void_p * max(1, layout.n_buckets))()
    for b, e in enumerate(ready_events):
        if e.cuda_event == 0:
            raise ValueError(f"ready event of bucket {b} was never recorded")
        handles[b] = e.cuda_event
    h = hp.c()
    if group is None:
        _check(_abi.lib().zero_step_overlapped(layout.handle, handles, _ptr(grads),
                                               _stride(grads, layout, rank_stride), _ptr(master), _ptr(m), _ptr(v),
                                               _ptr(p16_shard), _ptr(p16_full), ctypes.byref(h), _ptr(nonfinite),
                                               _stream(stream)), "zero_step_overlapped")
    else:
        _check(_abi.lib().zero_step_overlapped_grouped(layout.handle, handles, int(group), _ptr(grads),
                                                       _stride(grads, layout, rank_stride), _ptr(master), _ptr(m),
                                                       _ptr(v), _ptr(p16_shard), _ptr(p16_full), ctypes.byref(h),
                                                       _ptr(nonfinite), _stream(stream)),
               "zero_step_overlapped_grouped")


class LossScaler:
    """Dynamic loss scaling state (zero_loss_scaler); advanced by step_dynamic() and
    step_dynamic_commit(), or by advance() where the caller decides the step."""

    def __init__(self, scale, factor=2.0, window=1000, min_scale=1.0):
        self.c = _abi.LossScaler(float(scale), float(factor), int(window), float(min_scale), 0, 0, 0)

    def __getattr__(self, name):
        return getattr(self.__dict__["c"], name)

    def advance(self, applied):
        """zero_loss_scaler_advance: count an applied step, or back off after a skipped one."""
        _check(_abi.lib().zero_loss_scaler_advance(ctypes.byref(self.c), int(bool(applied))),
               "zero_loss_scaler_advance")


def step_dynamic(layout, grads, reduced, master, m, v, p16_shard, p16_full, hp, scaler, nonfinite,
                 rank_stride=None, stream=None):
    """One step under dynamic loss scaling; returns True if the update was applied."""
    h = hp.c()
    applied = ctypes.c_int32(0)
    _check(_abi.lib().zero_step_dynamic(layout.handle, _ptr(grads), _stride(grads, layout, rank_stride),
                                        _ptr(reduced), _ptr(master), _ptr(m), _ptr(v), _ptr(p16_shard),
                                        _ptr(p16_full), ctypes.byref(h), ctypes.byref(scaler.c), _ptr(nonfinite),
                                        ctypes.byref(applied), _stream(stream)), "zero_step_dynamic")
    return bool(applied.value)


def step_dynamic_commit(layout, grads, state_in, state_out, p16_out, p16_full, hp, scaler, nonfinite,
                        rank_stride=None, stream=None):
    """zero_step_dynamic_commit: state_in / state_out are (master, m, v) triples.  Returns
    True if the step was applied (then state_out and p16_out are the new current set)."""
    h = hp.c()
    applied = ctypes.c_int32(0)
    (mi, m_i, vi), (mo, m_o, vo) = state_in, state_out
    _check(_abi.lib().zero_step_dynamic_commit(layout.handle, _ptr(grads), _stride(grads, layout, rank_stride),
                                               _ptr(mi), _ptr(m_i), _ptr(vi), _ptr(mo), _ptr(m_o), _ptr(vo),
                                               _ptr(p16_out), _ptr(p16_full), ctypes.byref(h),
                                               ctypes.byref(scaler.c), _ptr(nonfinite), ctypes.byref(applied),
                                               _stream(stream)), "zero_step_dynamic_commit")
    return bool(applied.value)


def step_host(layout, grads_host, grads_dev, master, m, v, p16_shard, p16_full, p16_host, hp,
              nonfinite=None, rank_stride=None, stream=None):
    """grads_host / p16_host: page-locked (pinned) host tensors."""
    h = hp.c()
    _check(_abi.lib().zero_step_host(layout.handle, _ptr(grads_host), _ptr(grads_dev),
                                     _stride(grads_dev, layout, rank_stride), _ptr(master), _ptr(m), _ptr(v),
                                     _ptr(p16_shard), _ptr(p16_full), _ptr(p16_host), ctypes.byref(h),
                                     _ptr(nonfinite), _stream(stream)), "zero_step_host")


def step_noalloc(layout, grads, master, m, v, p16_shard, p16_full, hp, nonfinite=None, rank_stride=None,
                 stream=None):
    """zero_step for callers that cannot allocate device memory: same result, with the
    step's scratch in the library's static device array (at most
    _abi.NOALLOC_MAX_SEGMENTS segments; calls that overlap on the GPU race).  The layout
    need not be uploaded with to_device()."""
    h = hp.c()
    _check(_abi.lib().zero_step_noalloc(layout.handle, _ptr(grads), _stride(grads, layout, rank_stride),
                                        _ptr(master), _ptr(m), _ptr(v), _ptr(p16_shard), _ptr(p16_full),
                                        ctypes.byref(h), _ptr(nonfinite), _stream(stream)), "zero_step_noalloc")


def _ptr_array(ptrs):
    arr = (ctypes.c_void_p * max(1, len(ptrs)))()
    for i, p in enumerate(ptrs):
        arr[i] = _ptr(p)
    return arr


def step_ranks(layout, rank_grads, master, m, v, p16_shard, p16_full, hp, nonfinite=None, stream=None):
    """zero_step with rank r's gradients in rank_grads[r] (tensors or device addresses)."""
    h = hp.c()
    _check(_abi.lib().zero_step_ranks(layout.handle, _ptr_array(rank_grads), _ptr(master), _ptr(m), _ptr(v),
                                      _ptr(p16_shard), _ptr(p16_full), ctypes.byref(h), _ptr(nonfinite),
                                      _stream(stream)), "zero_step_ranks")


def step_shard(layout, shard, rank_grads, master_k, m_k, v_k, p16_out, hp, nonfinite=None, stream=None):
    """The update of one shard with shard-local state (zero_step_shard)."""
    h = hp.c()
    _check(_abi.lib().zero_step_shard(layout.handle, int(shard), _ptr_array(rank_grads), _ptr(master_k), _ptr(m_k),
                                      _ptr(v_k), _ptr(p16_out), ctypes.byref(h), _ptr(nonfinite), _stream(stream)),
           "zero_step_shard")


def step_shard_commit(layout, shard, rank_grads, state_in, state_out, p16_out, hp, scaler, nonfinite,
                      stream=None):
    """zero_step_shard_commit: shard `shard`'s update from state_in into state_out ((master,
    m, v) triples of [S] buffers) at the scaler's scale and step; returns the shard's count
    of non-finite reduced gradients (the stream is synchronised).  The scaler is not
    advanced: the ranks decide together."""
    h = hp.c()
    total = ctypes.c_int64(0)
    (mi, m_i, vi), (mo, m_o, vo) = state_in, state_out
    _check(_abi.lib().zero_step_shard_commit(layout.handle, int(shard), _ptr_array(rank_grads), _ptr(mi), _ptr(m_i),
                                             _ptr(vi), _ptr(mo), _ptr(m_o), _ptr(vo), _ptr(p16_out), ctypes.byref(h),
                                             ctypes.byref(scaler.c), _ptr(nonfinite), ctypes.byref(total),
                                             _stream(stream)), "zero_step_shard_commit")
    return int(total.value)


def copy_shard(layout, shard, src, dst, stream=None):
    _check(_abi.lib().zero_copy_shard(layout.handle, int(shard), _ptr(src), _ptr(dst), _stream(stream)),
           "zero_copy_shard")


def ipc_handle(tensor_or_ptr):
    """(64-byte CUDA IPC handle of the allocation holding the pointer, byte offset)."""
    buf = ctypes.create_string_buffer(64)
    off = ctypes.c_int64(0)
    _check(_abi.lib().zero_ipc_get_handle(_ptr(tensor_or_ptr), buf, ctypes.byref(off)), "zero_ipc_get_handle")
    return buf.raw, off.value


def ipc_open(handle):
    """Map another process's (handle, offset); returns the device address in this process."""
    raw, off = handle
    p = ctypes.c_void_p()
    _check(_abi.lib().zero_ipc_open(ctypes.create_string_buffer(bytes(raw), 64), int(off), ctypes.byref(p)),
           "zero_ipc_open")
    return p.value, int(off)


def ipc_close(mapped):
    """Unmap what ipc_open returned."""
    ptr, off = mapped
    _check(_abi.lib().zero_ipc_close(ptr, off), "zero_ipc_close")


def get_error(layout, stream=None):
    _check(_abi.lib().zero_get_error(layout.handle, _stream(stream)), "zero_get_error")
