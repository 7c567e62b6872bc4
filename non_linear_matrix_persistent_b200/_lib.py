"""ctypes view of libm2rnn.so (declared in include/m2rnn.h).

The library is the only implementation of the recurrence in this package:
if it is missing or fails to load, every call raises.  There is no CPU
fallback.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libm2rnn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_MISALIGNED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_TIMEOUT = range(7)
MODE_BF16_TC, MODE_FP32_DEBUG, MODE_BF16_TC_FAST_TANH, MODE_BF16_MMA_SYNC = 0, 1, 2, 3

# Every entry point declared in include/m2rnn.h.
EXPORTS = ("m2rnn_workspace_size", "m2rnn_forward", "m2rnn_backward", "m2rnn_backward_noalloc",
           "m2rnn_get_device_status", "m2rnn_status_string", "m2rnn_set_wait_limit_ns",
           "m2rnn_debug_set_fault")


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int), ("K", ctypes.c_int),
                ("V", ctypes.c_int), ("mode", ctypes.c_int), ("ckpt_stride", ctypes.c_int),
                ("qk_heads", ctypes.c_int), ("f_is_logit", ctypes.c_int)]


class M2RNNError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s" % (what, status_string(status)))


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libm2rnn.so not built (run non_linear_matrix_persistent_b200/build.py): %s" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i, P = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.POINTER(Dims)
        L.m2rnn_workspace_size.argtypes = [P, i]
        L.m2rnn_workspace_size.restype = sz
        L.m2rnn_forward.argtypes = [P] + [vp] * 10 + [sz, vp]
        L.m2rnn_forward.restype = i
        L.m2rnn_backward.argtypes = [P] + [vp] * 15 + [sz, vp]
        L.m2rnn_backward.restype = i
        L.m2rnn_backward_noalloc.argtypes = [P] + [vp] * 14 + [vp]
        L.m2rnn_backward_noalloc.restype = i
        L.m2rnn_get_device_status.argtypes = [vp, vp]
        L.m2rnn_get_device_status.restype = i
        L.m2rnn_status_string.argtypes = [i]
        L.m2rnn_status_string.restype = ctypes.c_char_p
        L.m2rnn_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.m2rnn_set_wait_limit_ns.restype = None
        L.m2rnn_debug_set_fault.argtypes = [i]
        L.m2rnn_debug_set_fault.restype = i
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().m2rnn_status_string(int(s)).decode()
