"""Python binding of libqgalore.so, the B200 (sm_100a) Q-GaLore optimizer-step library.

Argument marshalling only: every function forwards to the C ABI declared in
include/qgalore.h under the same name.  The library is loaded on first use and
its absence is an error (there is no fallback).  Device buffers are passed as
integer addresses (e.g. ``tensor.data_ptr()``) and streams as integer handles
(e.g. ``torch.cuda.current_stream().cuda_stream``).
"""
from __future__ import annotations

import ctypes
import os
from ctypes import (POINTER, Structure, byref, c_char_p, c_double, c_float, c_int32, c_int64, c_size_t,
                    c_uint32, c_uint64, c_void_p)

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqgalore.so")

QG_OK, QG_EINVAL, QG_ESHAPE, QG_EALIGN, QG_ESTATE, QG_ECUDA, QG_ETIMEOUT, QG_ENONFINITE = range(8)


class QGError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__(f"{where}: {qg_status_str(status)} ({status})" if where else qg_status_str(status))


class qg_config(Structure):
    _fields_ = [("m", c_int32), ("n", c_int32), ("r", c_int32), ("w_group", c_int32), ("p_group", c_int32),
                ("mom_block", c_int32), ("beta1", c_float), ("beta2", c_float), ("eps", c_float), ("lr", c_float),
                ("alpha", c_float), ("gamma", c_float), ("delta0", c_int32), ("oversample", c_int32),
                ("power_iters", c_int32), ("seed", c_uint64), ("layer_id", c_uint32), ("mom_refresh", c_int32),
                ("proj_side", c_int32), ("w_rescale", c_int32)]


class qg_layer_views(Structure):
    _fields_ = [("status", c_void_p), ("Pq", c_void_p), ("sP", c_void_p), ("Pq_prev", c_void_p),
                ("sP_prev", c_void_p), ("Mq", c_void_p), ("Vq", c_void_p), ("sM", c_void_p), ("sV", c_void_p),
                ("ld_mom", c_int64), ("nblk", c_int32), ("p_rows", c_int32), ("mom_rows", c_int32),
                ("mom_cols", c_int32)]


class qg_sched(Structure):
    _fields_ = [("t", c_int64), ("delta", c_int32), ("t_next", c_int64), ("n_refresh", c_int32),
                ("has_projection", c_int32)]


class qg_refresh_info(Structure):
    _fields_ = [("refreshed", c_int32), ("has_cossim", c_int32), ("cossim", c_float), ("delta", c_int32),
                ("t_next", c_int64), ("n_refresh", c_int32)]


class qg_kernel_times(Structure):
    _fields_ = [("launches", c_int64), ("device_ms", c_double), ("flops", c_double), ("bytes", c_double)]


(QG_KERNEL_DEQUANT, QG_KERNEL_PROJECT_ADAM, QG_KERNEL_BACKPROJECT_SR, QG_KERNEL_OTHER, QG_KERNEL_LINEAR_DEQUANT,
 QG_KERNEL_LINEAR_GEMM, QG_KERNEL_LINEAR_FUSED, QG_KERNEL_KINDS) = range(8)

_SIGNATURES = {
    "qg_status_str": (c_char_p, [c_int32]),
    "qg_config_default": (None, [POINTER(qg_config), c_int32, c_int32, c_int32]),
    "qg_state_bytes": (c_size_t, [POINTER(qg_config)]),
    "qg_step_workspace_bytes": (c_size_t, [POINTER(qg_config)]),
    "qg_refresh_workspace_bytes": (c_size_t, [POINTER(qg_config)]),
    "qg_layer_init": (c_int32, [POINTER(c_void_p), POINTER(qg_config), c_void_p, c_size_t, c_void_p, c_int64,
                                c_void_p, c_void_p]),
    "qg_layer_destroy": (c_int32, [c_void_p]),
    "qg_layer_views_get": (c_int32, [c_void_p, POINTER(qg_layer_views)]),
    "qg_layer_sched_get": (c_int32, [c_void_p, POINTER(qg_sched)]),
    "qg_layer_sched_set": (c_int32, [c_void_p, POINTER(qg_sched)]),
    "qg_layer_set_projection": (c_int32, [c_void_p, c_void_p, c_void_p, c_int32, c_void_p]),
    "qg_step": (c_int32, [c_void_p, c_void_p, c_int64, c_void_p, c_size_t, c_void_p]),
    "qg_step_noalloc": (c_int32, [c_void_p, c_void_p, c_int64, c_void_p]),
    "qg_step_batch": (c_int32, [POINTER(c_void_p), POINTER(c_void_p), POINTER(c_int64), c_int32, c_void_p, c_size_t,
                                c_void_p]),
    "qg_step_batch_workspace_bytes": (c_size_t, [POINTER(POINTER(qg_config)), c_int32]),
    "qg_refresh": (c_int32, [c_void_p, c_void_p, c_int64, c_int32, c_void_p, c_size_t, POINTER(qg_refresh_info),
                             c_void_p]),
    "qg_cossim_workspace_bytes": (c_size_t, [c_int32, c_int32]),
    "qg_cossim": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_int64, c_void_p, c_void_p, c_size_t, c_void_p]),
    "qg_layer_status": (c_int32, [c_void_p, c_void_p]),
    "qg_sched_after_refresh": (c_int32, [c_int64, c_int32, c_int32, c_float, c_float, POINTER(c_int32),
                                         POINTER(c_int64)]),
    "qg_quantize_projection": (c_int32, [c_void_p, c_int64, c_int32, c_int32, c_void_p, c_void_p, c_void_p]),
    "qg_profile_enable": (c_int32, [c_int32]),
    "qg_profile_collect": (c_int32, [POINTER(qg_kernel_times), c_int32]),
    "qg_philox4x32_10": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_uint32, c_uint32, c_void_p,
                                   c_void_p]),
    "qg_dequant_projection": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_void_p]),
    "qg_gemm_bf16": (c_int32, [c_void_p, c_int64, c_int32, c_void_p, c_int64, c_int32, c_void_p, c_int64, c_int32,
                               c_int32, c_int32, c_void_p]),
    "qg_selfcheck_exact_math": (c_int32, [c_int32, c_uint64, c_uint64, c_void_p, c_void_p]),
    "qg_selfcheck_wait_timeout": (c_int32, [c_uint64, c_void_p, c_void_p, c_void_p]),
    "qg_linear_dequant_weight": (c_int32, [c_void_p, c_int64, c_void_p, c_int32, c_int32, c_void_p, c_int64,
                                           c_void_p]),
    "qg_linear_forward": (c_int32, [c_void_p, c_int64, c_void_p, c_int64, c_int32, c_int32, c_int32, c_void_p,
                                    c_int64, c_void_p]),
    "qg_linear_forward_int8": (c_int32, [c_void_p, c_int64, c_void_p, c_int64, c_void_p, c_int32, c_int32, c_int32,
                                         c_void_p, c_int64, c_void_p]),
    "qg_linear_backward_data": (c_int32, [c_void_p, c_int64, c_void_p, c_int64, c_int32, c_int32, c_int32,
                                          c_void_p, c_int64, c_void_p]),
    "qg_linear_backward_weight": (c_int32, [c_void_p, c_int64, c_void_p, c_int64, c_int32, c_int32, c_int32,
                                            c_void_p, c_int64, c_void_p]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m quantized_rank_gradient_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def exported_symbols() -> list[str]:
    return list(_SIGNATURES)


def _forward(name):
    def f(*args):
        return getattr(lib(), name)(*args)
    f.__name__ = name
    f.__doc__ = f"Calls {name} of include/qgalore.h."
    return f


for _name in _SIGNATURES:
    globals()[_name] = _forward(_name)


def qg_status_str(status: int) -> str:  # noqa: F811 - decode the C string
    return lib().qg_status_str(int(status)).decode()


def check(status: int, where: str = "") -> None:
    """Raise QGError for a non-zero status."""
    if status != QG_OK:
        raise QGError(status, where)


def config(m: int, n: int, r: int, **kw) -> qg_config:
    """qg_config_default(m, n, r) with fields overridden by keyword."""
    c = qg_config()
    lib().qg_config_default(byref(c), m, n, r)
    for k, v in kw.items():
        setattr(c, k, v)
    return c
