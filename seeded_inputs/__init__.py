"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

Values are a pure function of (seed, stream, flat index) through Philox4x32-10 (see
philox.h), so the host fill (numpy arrays) and the device fill (torch CUDA tensors)
give identical bits, and a sampled check at full size can regenerate just the inputs
of the sampled elements.  Nothing here computes any part of the optimizer step.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_HOST = None
_CUDA = None

DEFAULT_SEED = 0x5EED
STREAM_MASTER = 1
STREAM_M = 2
STREAM_V = 3
STREAM_SIZES = 4
STREAM_GRAD0 = 1024

_i64 = ctypes.c_int64
_u32 = ctypes.c_uint32
_i32 = ctypes.c_int32
_dbl = ctypes.c_double
_vp = ctypes.c_void_p


def _host():
    global _HOST
    if _HOST is None:
        _build.build(cuda=False)
        lib = ctypes.CDLL(_build.HOST_LIB)
        lib.si_philox4x32_10_host.argtypes = [_vp, _vp, _vp]
        lib.si_f32_to_f16_host.argtypes = [_vp, _vp, _i64]
        lib.si_irwin_hall_host.argtypes = [_vp, _i64, _u32, _u32]
        lib.si_extra_words_host.argtypes = [_vp, _i64, _u32, _u32]
        lib.si_fill_f32_host.argtypes = [_vp, _i64, _i64, _u32, _u32, _dbl, ctypes.c_int]
        lib.si_gather_f32_host.argtypes = [_vp, _vp, _i64, _i64, _u32, _u32, _dbl, ctypes.c_int]
        lib.si_fill_grads_host.argtypes = [_vp, _i32, _i64, _i64, _u32, _dbl, _dbl, _u32, _dbl]
        lib.si_gather_grads_host.argtypes = [_vp, _vp, _i64, _i32, _i64, _u32, _dbl, _dbl, _u32, _dbl]
        _HOST = lib
    return _HOST


def _cuda():
    global _CUDA
    if _CUDA is None:
        _build.build()
        lib = ctypes.CDLL(_build.CUDA_LIB)
        lib.si_fill_f32_cuda.argtypes = [_vp, _i64, _i64, _u32, _u32, _dbl, ctypes.c_int, _vp]
        lib.si_fill_f32_cuda.restype = ctypes.c_int
        lib.si_fill_grads_cuda.argtypes = [_vp, _i32, _i64, _i64, _u32, _dbl, _dbl, _u32, _dbl, _vp]
        lib.si_fill_grads_cuda.restype = ctypes.c_int
        lib.si_fill_grads_range_cuda.argtypes = [_vp, _i32, _i64, _i64, _i64, _i64, _u32, _dbl, _dbl, _u32,
                                                 _dbl, _vp]
        lib.si_fill_grads_range_cuda.restype = ctypes.c_int
        _CUDA = lib
    return _CUDA


def _ptr(a):
    return a.ctypes.data_as(_vp)


def heavy_q32(frac):
    """Threshold on a uniform 32-bit word selecting a fraction `frac` of entries."""
    return int(round(frac * 2.0 ** 32)) if frac else 0


# ---------------------------------------------------------------- host (numpy)

def philox4x32_10(ctr, key):
    c = np.asarray(ctr, dtype=np.uint32)
    k = np.asarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    _host().si_philox4x32_10_host(_ptr(c), _ptr(k), _ptr(out))
    return out


def f32_to_f16_bits(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(x.shape, dtype=np.uint16)
    _host().si_f32_to_f16_host(_ptr(x), _ptr(out), x.size)
    return out


def irwin_hall(n, seed, stream):
    out = np.zeros(n, dtype=np.int32)
    _host().si_irwin_hall_host(_ptr(out), n, seed, stream)
    return out


def extra_words(n, seed, stream):
    out = np.zeros(n, dtype=np.uint32)
    _host().si_extra_words_host(_ptr(out), n, seed, stream)
    return out


def fill_f32(n, valid, seed, stream, sigma, absval=False):
    out = np.empty(n, dtype=np.float32)
    _host().si_fill_f32_host(_ptr(out), n, valid, seed, stream, sigma, int(absval))
    return out


def gather_f32(idx, valid, seed, stream, sigma, absval=False):
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.empty(idx.size, dtype=np.float32)
    _host().si_gather_f32_host(_ptr(out), _ptr(idx), idx.size, valid, seed, stream, sigma, int(absval))
    return out


def fill_grads(n_ranks, rank_stride, valid, seed, sigma, loss_scale, heavy_frac=0.0, heavy_mult=1.0):
    """fp16 bit patterns, shape [n_ranks, rank_stride]."""
    out = np.empty((n_ranks, rank_stride), dtype=np.uint16)
    _host().si_fill_grads_host(_ptr(out), n_ranks, rank_stride, valid, seed, sigma, loss_scale,
                               heavy_q32(heavy_frac), heavy_mult)
    return out


def gather_grads(idx, n_ranks, valid, seed, sigma, loss_scale, heavy_frac=0.0, heavy_mult=1.0):
    """fp16 bit patterns, shape [len(idx), n_ranks]."""
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.empty((idx.size, n_ranks), dtype=np.uint16)
    _host().si_gather_grads_host(_ptr(out), _ptr(idx), idx.size, n_ranks, valid, seed, sigma,
                                 loss_scale, heavy_q32(heavy_frac), heavy_mult)
    return out


# ---------------------------------------------------------------- device (torch)

def _check(err, what):
    if err != 0:
        raise RuntimeError(f"{what}: CUDA error {err}")


def fill_f32_cuda(t, valid, seed, stream, sigma, absval=False, cuda_stream=None):
    import torch
    s = cuda_stream if cuda_stream is not None else torch.cuda.current_stream(t.device).cuda_stream
    assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
    _check(_cuda().si_fill_f32_cuda(t.data_ptr(), t.numel(), valid, seed, stream, sigma,
                                    int(absval), s), "si_fill_f32_cuda")


def fill_grads_cuda(t, valid, seed, sigma, loss_scale, heavy_frac=0.0, heavy_mult=1.0, cuda_stream=None):
    """t: CUDA int16/uint16 tensor [n_ranks, rank_stride] receiving fp16 bit patterns."""
    import torch
    s = cuda_stream if cuda_stream is not None else torch.cuda.current_stream(t.device).cuda_stream
    assert t.is_cuda and t.dim() == 2 and t.is_contiguous() and t.element_size() == 2
    _check(_cuda().si_fill_grads_cuda(t.data_ptr(), t.shape[0], t.shape[1], valid, seed, sigma,
                                      loss_scale, heavy_q32(heavy_frac), heavy_mult, s),
           "si_fill_grads_cuda")


def fill_grads_range_cuda(t, lo, hi, valid, seed, sigma, loss_scale, heavy_frac=0.0, heavy_mult=1.0,
                          cuda_stream=None):
    """Fill flat indices [lo, hi) of every rank's row of t [n_ranks, rank_stride]."""
    import torch
    s = cuda_stream if cuda_stream is not None else torch.cuda.current_stream(t.device).cuda_stream
    assert t.is_cuda and t.dim() == 2 and t.is_contiguous() and t.element_size() == 2
    _check(_cuda().si_fill_grads_range_cuda(t.data_ptr(), t.shape[0], t.shape[1], lo, hi, valid, seed, sigma,
                                            loss_scale, heavy_q32(heavy_frac), heavy_mult, s),
           "si_fill_grads_range_cuda")
