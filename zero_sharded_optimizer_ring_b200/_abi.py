"""ctypes declarations of the C ABI in include/zero.h (argument marshalling only)."""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# ZERO_B200_DEBUG=1 selects the bounds-checking build (libzero_b200_debug.so, same ABI)
DEBUG = os.environ.get("ZERO_B200_DEBUG", "") == "1"
LIB_PATH = os.path.join(_HERE, "libzero_b200_debug.so" if DEBUG else "libzero_b200.so")

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_p_i64 = ctypes.POINTER(ctypes.c_int64)

ZERO_OK = 0
NOALLOC_MAX_SEGMENTS = 8191   # ZERO_NOALLOC_MAX_SEGMENTS in include/zero.h
OVERLAP_PLANS = 5             # ZERO_OVERLAP_PLANS in include/zero.h
STATUS_NAMES = {0: "ZERO_OK", 1: "ZERO_ERR_INVALID", 2: "ZERO_ERR_ALIGN", 3: "ZERO_ERR_CUDA",
                4: "ZERO_ERR_OOM", 5: "ZERO_ERR_TIMEOUT", 6: "ZERO_ERR_STATE", 7: "ZERO_ERR_BOUNDS"}


class LayoutDesc(ctypes.Structure):
    _fields_ = [("n_ranks", _i32), ("stage", _i32), ("n_tensors", _i64),
                ("tensor_numel", _p_i64), ("bucket_elems", _i64), ("pad_align", _i64),
                ("n_units", _i64), ("unit_first_tensor", _p_i64), ("wire_fp16", _i32)]


class LayoutInfo(ctypes.Structure):
    _fields_ = [("psi", _i64), ("shard", _i64), ("padded", _i64), ("n_buckets", _i64),
                ("n_segments", _i64), ("n_units", _i64), ("tile_elems", _i64), ("n_tiles", _i64)]


class AdamWHparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double), ("beta2", ctypes.c_double),
                ("eps", ctypes.c_double), ("weight_decay", ctypes.c_double),
                ("loss_scale", ctypes.c_double), ("step", _i64)]


class Counters(ctypes.Structure):
    _fields_ = [("mem_p16", _i64), ("mem_g16", _i64), ("mem_os", _i64), ("mem_total", _i64),
                ("sent_elems", _i64), ("recv_elems", _i64)]


class LossScaler(ctypes.Structure):
    _fields_ = [("scale", ctypes.c_double), ("factor", ctypes.c_double), ("window", _i64),
                ("min_scale", ctypes.c_double), ("clean_steps", _i64), ("step", _i64), ("skipped", _i64)]


class StepScalars(ctypes.Structure):
    _fields_ = [(n, ctypes.c_float) for n in ("inv_scale", "decay", "beta1", "omb1", "beta2", "omb2",
                                              "step_size", "sqrt_bc2", "eps")]


class StepEvents(ctypes.Structure):
    _fields_ = [("update_begin", _vp), ("update_end", _vp), ("gather_begin", _vp), ("gather_end", _vp)]


# name -> (restype, argtypes); every function declared in include/zero.h
SIGNATURES = {
    "zero_layout_create": (_i32, [ctypes.POINTER(LayoutDesc), ctypes.POINTER(_vp)]),
    "zero_layout_destroy": (None, [_vp]),
    "zero_layout_get_info": (_i32, [_vp, ctypes.POINTER(LayoutInfo)]),
    "zero_layout_get_tables": (_i32, [_vp, _vp, _vp, _vp, _vp]),
    "zero_layout_counters": (_i32, [_vp, ctypes.POINTER(Counters)]),
    "zero_layout_to_device": (_i32, [_vp, _vp]),
    "zero_layout_device_segments": (_i32, [_vp, _vp, _vp]),
    "zero_reduce_scatter": (_i32, [_vp, _i64, _vp, _i64, _vp, _vp, _vp]),
    "zero_adamw_shard_step": (_i32, [_vp, _i32, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(AdamWHparams), _vp]),
    "zero_allgather": (_i32, [_vp, _i64, _vp, _vp, _vp]),
    "zero_gather_unit": (_i32, [_vp, _i64, _vp, _vp, _vp]),
    "zero_step": (_i32, [_vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(AdamWHparams), _vp,
                         ctypes.POINTER(StepEvents), _vp]),
    "zero_step_scalars_fill": (_i32, [_vp, ctypes.POINTER(AdamWHparams), ctypes.POINTER(StepScalars)]),
    "zero_step_device_scalars": (_i32, [_vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "zero_step_bucket": (_i32, [_vp, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(AdamWHparams),
                                _vp, _vp]),
    "zero_step_overlapped": (_i32, [_vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(AdamWHparams),
                                    _vp, _vp]),
    "zero_overlap_plan": (_i32, [_vp, ctypes.POINTER(_i32), _vp]),
    "zero_step_overlapped_grouped": (_i32, [_vp, _vp, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _vp,
                                            ctypes.POINTER(AdamWHparams), _vp, _vp]),
    "zero_step_dynamic": (_i32, [_vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(AdamWHparams),
                                 ctypes.POINTER(LossScaler), _vp, ctypes.POINTER(_i32), _vp]),
    "zero_step_dynamic_commit": (_i32, [_vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                        ctypes.POINTER(AdamWHparams), ctypes.POINTER(LossScaler), _vp,
                                        ctypes.POINTER(_i32), _vp]),
    "zero_step_host": (_i32, [_vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp,
                              ctypes.POINTER(AdamWHparams), _vp, _vp]),
    "zero_step_noalloc": (_i32, [_vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(AdamWHparams), _vp, _vp]),
    "zero_step_ranks": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(AdamWHparams), _vp, _vp]),
    "zero_step_shard": (_i32, [_vp, _i32, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(AdamWHparams), _vp, _vp]),
    "zero_step_shard_commit": (_i32, [_vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                      ctypes.POINTER(AdamWHparams), ctypes.POINTER(LossScaler), _vp,
                                      ctypes.POINTER(_i64), _vp]),
    "zero_loss_scaler_advance": (_i32, [ctypes.POINTER(LossScaler), _i32]),
    "zero_copy_shard": (_i32, [_vp, _i32, _vp, _vp, _vp]),
    "zero_ipc_get_handle": (_i32, [_vp, _vp, ctypes.POINTER(_i64)]),
    "zero_ipc_open": (_i32, [_vp, _i64, ctypes.POINTER(_vp)]),
    "zero_ipc_close": (_i32, [_vp, _i64]),
    "zero_gather_unit_ranks": (_i32, [_vp, _i64, _vp, _vp, _vp]),
    "zero_set_impl": (_i32, [_vp, _i32]),
    "zero_set_max_ctas": (_i32, [_vp, _i32]),
    "zero_set_gather_ctas": (_i32, [_vp, _i32]),
    "zero_debug_set_wait": (_i32, [_vp, _i64, _i32]),
    "zero_get_error": (_i32, [_vp, _vp]),
    "zero_status_string": (ctypes.c_char_p, [_i32]),
}

_LIB = None


def lib():
    """Load libzero_b200.so.  There is no fallback: without the library nothing runs."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m zero_sharded_optimizer_ring_b200.build"
                              f"{' --debug' if DEBUG else ''}` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB
