"""ctypes view of ``libfastvim_ssm.so`` (the C ABI declared in ``include/fastvim_ssm.h``).

Argument marshalling only.  The library is loaded from this package directory; if it is missing
or fails to load, every call raises -- there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libfastvim_ssm.so")

FV_OK = 0
FV_ERR_NULL = 1
FV_ERR_SHAPE = 2
FV_ERR_ALIGN = 3
FV_ERR_INDEX = 4
FV_ERR_WORKSPACE = 5
FV_ERR_CUDA = 6
FV_ERR_TIMEOUT = 7
FV_ERR_UNSUPPORTED = 8
FV_ERR_ALIAS = 9

FV_FLAG_ZOH_EXACT = 1
FV_FLAG_PATH_STAGED = 2
FV_FLAG_PATH_FUSED = 4
FV_FLAG_TRACE = 8
FV_FLAG_LAYERNORM = 16
FV_FLAG_CONV_SILU = 32
FV_FLAG_KEEP_STATES = 64

# Every exported symbol of the ABI, as the header declares it.
EXPORTS = (
    "fastvim_status_string",
    "fastvim_last_error",
    "fastvim_abi_version",
    "fastvim_ssm_validate",
    "fastvim_ssm_workspace_size",
    "fastvim_ssm_workspace_layout",
    "fastvim_ssm_launch_count",
    "fastvim_ssm_launch_name",
    "fastvim_ssm_forward",
    "fastvim_ssm_forward_events",
    "fastvim_ssm_forward_host",
    "fastvim_ssm_forward_noalloc",
    "fastvim_selftest_bounded_wait",
    "fastvim_selftest_math",
    "fastvim_get_device_status",
    "fastvim_ssm_backward_workspace_size",
    "fastvim_ssm_backward_workspace_layout",
    "fastvim_ssm_backward_launch_count",
    "fastvim_ssm_backward_launch_name",
    "fastvim_ssm_backward",
    "fastvim_ssm_backward_events",
)


class FvSsmArgs(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("h", ctypes.c_int), ("w", ctypes.c_int), ("E", ctypes.c_int),
        ("N", ctypes.c_int), ("R", ctypes.c_int),
        ("pool_axis", ctypes.c_int),
        ("dir_flags", ctypes.c_uint),
        ("K", ctypes.c_int),
        ("pool_scale", ctypes.c_float),
        ("flags", ctypes.c_uint),
        ("x", ctypes.c_void_p), ("z", ctypes.c_void_p),
        ("A_log", ctypes.c_void_p), ("D", ctypes.c_void_p), ("W_x", ctypes.c_void_p),
        ("W_dt", ctypes.c_void_p), ("b_dt", ctypes.c_void_p),
        ("keep_idx", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
        ("ln_gamma", ctypes.c_void_p), ("ln_beta", ctypes.c_void_p), ("ln_eps", ctypes.c_float),
        ("d_conv", ctypes.c_int), ("conv_w", ctypes.c_void_p), ("conv_b", ctypes.c_void_p),
    ]


class FvWsLayout(ctypes.Structure):
    _fields_ = [
        ("total_bytes", ctypes.c_size_t), ("status", ctypes.c_size_t), ("xbar", ctypes.c_size_t),
        ("u", ctypes.c_size_t), ("ys", ctypes.c_size_t), ("row_of", ctypes.c_size_t),
        ("row_off", ctypes.c_size_t), ("row_tok", ctypes.c_size_t),
        ("delta", ctypes.c_size_t), ("ctrl", ctypes.c_size_t), ("trace", ctypes.c_size_t),
        ("trace_records", ctypes.c_size_t), ("ckpt", ctypes.c_size_t), ("scan_dt", ctypes.c_size_t),
        ("T", ctypes.c_int), ("S", ctypes.c_int), ("nd", ctypes.c_int),
    ]


class FvSsmGrads(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in ("dy", "dx", "dz", "dA_log", "dD", "dW_x", "dW_dt", "db_dt",
                                                     "dln_gamma", "dln_beta")]


class FvBwdWsLayout(ctypes.Structure):
    _fields_ = [(name, ctypes.c_size_t) for name in ("total_bytes", "dys", "dxbar", "du", "dxs", "ckpt", "status",
                                                     "delta", "partials")]


class FastvimError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = f"{where}: {status_string(status)}"
        if detail:
            msg += f" [{detail}]"
        super().__init__(msg)


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it is absent (build it with ``python -m
    pooled_selective_scan_b200.build``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: the FastVim SSM layer has no other "
                                  "implementation; build it with `python -m pooled_selective_scan_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P = ctypes.POINTER
            L.fastvim_status_string.argtypes = [ctypes.c_int]
            L.fastvim_status_string.restype = ctypes.c_char_p
            L.fastvim_last_error.argtypes = []
            L.fastvim_last_error.restype = ctypes.c_char_p
            L.fastvim_abi_version.argtypes = []
            L.fastvim_abi_version.restype = ctypes.c_int
            L.fastvim_ssm_validate.argtypes = [P(FvSsmArgs)]
            L.fastvim_ssm_validate.restype = ctypes.c_int
            L.fastvim_ssm_workspace_size.argtypes = [P(FvSsmArgs)]
            L.fastvim_ssm_workspace_size.restype = ctypes.c_size_t
            L.fastvim_ssm_workspace_layout.argtypes = [P(FvSsmArgs), P(FvWsLayout)]
            L.fastvim_ssm_workspace_layout.restype = ctypes.c_int
            L.fastvim_ssm_launch_count.argtypes = [P(FvSsmArgs)]
            L.fastvim_ssm_launch_count.restype = ctypes.c_int
            L.fastvim_ssm_launch_name.argtypes = [P(FvSsmArgs), ctypes.c_int]
            L.fastvim_ssm_launch_name.restype = ctypes.c_char_p
            L.fastvim_ssm_forward_events.argtypes = [P(FvSsmArgs), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                                     P(ctypes.c_void_p), ctypes.c_int]
            L.fastvim_ssm_forward_events.restype = ctypes.c_int
            L.fastvim_ssm_forward.argtypes = [P(FvSsmArgs), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
            L.fastvim_ssm_forward.restype = ctypes.c_int
            L.fastvim_ssm_forward_host.argtypes = [P(FvSsmArgs), P(FvSsmArgs), ctypes.c_void_p, ctypes.c_size_t,
                                                   ctypes.c_void_p]
            L.fastvim_ssm_forward_host.restype = ctypes.c_int
            L.fastvim_ssm_forward_noalloc.argtypes = [P(FvSsmArgs), ctypes.c_void_p]
            L.fastvim_ssm_forward_noalloc.restype = ctypes.c_int
            L.fastvim_selftest_bounded_wait.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint, ctypes.c_void_p]
            L.fastvim_selftest_bounded_wait.restype = ctypes.c_int
            L.fastvim_selftest_math.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                                ctypes.c_void_p]
            L.fastvim_selftest_math.restype = ctypes.c_int
            L.fastvim_get_device_status.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
            L.fastvim_get_device_status.restype = ctypes.c_int
            L.fastvim_ssm_backward_workspace_size.argtypes = [P(FvSsmArgs)]
            L.fastvim_ssm_backward_workspace_size.restype = ctypes.c_size_t
            L.fastvim_ssm_backward_workspace_layout.argtypes = [P(FvSsmArgs), P(FvBwdWsLayout)]
            L.fastvim_ssm_backward_workspace_layout.restype = ctypes.c_int
            L.fastvim_ssm_backward_launch_count.argtypes = [P(FvSsmArgs)]
            L.fastvim_ssm_backward_launch_count.restype = ctypes.c_int
            L.fastvim_ssm_backward_launch_name.argtypes = [P(FvSsmArgs), ctypes.c_int]
            L.fastvim_ssm_backward_launch_name.restype = ctypes.c_char_p
            L.fastvim_ssm_backward.argtypes = [P(FvSsmArgs), P(FvSsmGrads), ctypes.c_void_p, ctypes.c_size_t,
                                               ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
            L.fastvim_ssm_backward.restype = ctypes.c_int
            L.fastvim_ssm_backward_events.argtypes = [P(FvSsmArgs), P(FvSsmGrads), ctypes.c_void_p, ctypes.c_size_t,
                                                      ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                                      P(ctypes.c_void_p), ctypes.c_int]
            L.fastvim_ssm_backward_events.restype = ctypes.c_int
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().fastvim_status_string(int(status)).decode()


def last_error() -> str:
    return lib().fastvim_last_error().decode()


def check(status: int, where: str):
    if status != FV_OK:
        raise FastvimError(status, where, last_error() if status == FV_ERR_CUDA else "")
    return status
