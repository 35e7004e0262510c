"""ctypes loader for libhyena_b200.so (the C ABI declared in include/hyena.h).

The shared library is built in-tree (``python -m hyena_long_convolution_b200.build``).
There is no fallback: if the library is missing or cannot be loaded, every
entry point raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

SO = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhyena_b200.so")

STATUS = {
    0: "HYENA_OK",
    1: "HYENA_ERR_INVALID_ARG",
    2: "HYENA_ERR_ALIGNMENT",
    3: "HYENA_ERR_UNSUPPORTED",
    4: "HYENA_ERR_CUDA",
    5: "HYENA_ERR_TIMEOUT",
    6: "HYENA_ERR_WORKSPACE",
}

# name -> (restype, argtypes), mirroring include/hyena.h
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
SIGNATURES = {
    "hyena_status_string": (ctypes.c_char_p, [_I]),
    "hyena_abi_version": (_I, []),
    "hyena_last_launch_count": (_I, []),
    "hyena_last_error_message": (ctypes.c_char_p, []),
    "hyena_short_conv": (_I, [_P, _P, _P, _I64, _P, _P, _P, _I64, _P, _P, _I, _I, _I, _I, _P]),
    "hyena_short_conv_dft": (_I, [_P, _P, _P, _I64, _P, _P, _P, _I64, _P, _P, _I, _I, _I, _I, _P]),
    "hyena_modal_long_conv_workspace_size": (_SZ, [_I, _I, _I]),
    "hyena_modal_workspace_init": (_I, [_P, _SZ, _P]),
    "hyena_modal_long_conv": (_I, [_P, _P, _P, _I64, _P, _P, _P, _P, _I64, _P, _P,
                                   _I, _I, _I, _I, _P, _SZ, _P]),
    "hyena_modal_long_conv_noalloc": (_I, [_P, _P, _P, _I64, _P, _P, _P, _P, _I64, _P, _P,
                                           _I, _I, _I, _I, _P]),
    "hyena_modal_prepare": (_I, [_P, _P, _P, _I, _I, _I, _P, _SZ, _P]),
    "hyena_modal_long_conv_prepared": (_I, [_P, _P, _P, _I64, _P, _I64, _P, _P, _I, _I, _I, _I, _P, _SZ, _P]),
    "hyena_modal_host_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "hyena_modal_long_conv_host": (_I, [_P, _P, _P, _I64, _P, _P, _P, _P, _I64, _P, _P,
                                        _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "hyena_short_host_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "hyena_short_conv_host": (_I, [_P, _P, _P, _I64, _P, _P, _P, _I64, _P, _P, _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "hyena_modal_noalloc_check": (_I, [_P]),
    "hyena_modal_noalloc_scratch": (_I, [_P, _P]),
    "hyena_modal_decode": (_I, [_P, _P, _P, _I64, _P, _P, _P, _P, _I64, _P, _I, _I, _I, _P]),
    "hyena_short_decode": (_I, [_P, _P, _P, _I64, _P, _P, _P, _I64, _P, _I, _I, _I, _P]),
    "hyena_short_conv_packed": (_I, [_P, _I64, _I, _P, _P, _P, _I64, _P, _P, _I, _I, _I, _I, _P]),
    "hyena_modal_long_conv_packed": (_I, [_P, _I64, _I, _P, _P, _P, _P, _I64, _P, _P,
                                          _I, _I, _I, _I, _P, _SZ, _P]),
    "hyena_modal_decode_packed": (_I, [_P, _I64, _I, _P, _P, _P, _P, _I64, _P, _I, _I, _I, _P]),
    "hyena_short_decode_packed": (_I, [_P, _I64, _I, _P, _P, _P, _I64, _P, _I, _I, _I, _P]),
    "hyena_modal_long_conv_complex": (_I, [_P, _P, _P, _I64, _P, _P, _P, _P, _I64, _P, _P,
                                           _I, _I, _I, _I, _P, _SZ, _P]),
    "hyena_modal_decode_complex": (_I, [_P, _P, _P, _I64, _P, _P, _P, _P, _I64, _P, _I, _I, _I, _P]),
    "hyena_modal_long_conv_complex_packed": (_I, [_P, _I64, _I, _P, _P, _P, _P, _I64, _P, _P,
                                                  _I, _I, _I, _I, _P, _SZ, _P]),
    "hyena_modal_decode_complex_packed": (_I, [_P, _I64, _I, _P, _P, _P, _P, _I64, _P, _I, _I, _I, _P]),
    "hyena_modal_state_init": (_I, [_P, _I, _I, _I, _P]),
    "hyena_workspace_check": (_I, [_P, _P]),
}

_lock = threading.Lock()
_lib = None


class HyenaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")
        self.status = status


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(SO):
                raise ImportError(
                    f"{SO} is missing: build it with `python -m hyena_long_convolution_b200.build`")
            h = ctypes.CDLL(SO)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(h, name)
                f.restype = res
                f.argtypes = args
            _lib = h
    return _lib


def check(fn: str, status: int) -> None:
    if status != 0:
        err = HyenaError(fn, status)
        if status == 4:  # HYENA_ERR_CUDA: attach the failing runtime call
            err.args = (f"{err.args[0]} ({lib().hyena_last_error_message().decode()})",)
        raise err
