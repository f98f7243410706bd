"""ctypes loader for libfa2.so (C ABI in include/fa2.h).

Loading fails loudly: if the library is missing the caller gets an error that
says how to build it; nothing falls back to another implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

FA2_BF16 = 0
FA2_FP32 = 1
FA2_FP16 = 2

FA2_OK = 0
FA2_ERR_DEVICE_TIMEOUT = 8

FA2_BWD_DETERMINISTIC = 1
FA2_BWD_ONE_PASS = 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libfa2.so")
_lib: Optional[ctypes.CDLL] = None
_lock = threading.Lock()

# Every function the header declares, with its ctypes signature.
SIGNATURES = {
    "fa2_forward": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int] * 5
                    + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p]),
    "fa2_forward_ex": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int] * 7
                       + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p]),
    "fa2_backward_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int] * 5),
    "fa2_backward_workspace_bytes_ex": (ctypes.c_size_t, [ctypes.c_int] * 7),
    "fa2_backward_ex": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_int] * 7
                        + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                           ctypes.c_void_p]),
    "fa2_forward_block_sparse": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int] * 7
                                 + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]),
    "fa2_backward_block_sparse": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_int] * 7
                                  + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_size_t, ctypes.c_void_p]),
    "fa2_backward": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_int] * 5
                     + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                        ctypes.c_void_p]),
    "fa2_backward_timed": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_int] * 5
                           + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                              ctypes.c_void_p, ctypes.c_void_p]),
    "fa2_backward_opts": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_int] * 7
                          + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_uint,
                             ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "fa2_backward_noalloc": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_int] * 5
                             + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p]),
    "fa2_last_device_status": (ctypes.c_int, []),
    "fa2_clear_device_status": (ctypes.c_int, []),
    "fa2_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "fa2_watchdog_selftest": (ctypes.c_int, [ctypes.c_ulonglong, ctypes.c_void_p]),
}


class FA2Error(RuntimeError):
    def __init__(self, code: int):
        self.code = int(code)
        super().__init__(status_string(code))


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(_LIB_PATH):
                    raise ImportError(
                        f"{_LIB_PATH} is missing; build it with "
                        "`python -m causal_attention_fa2_b200.build` (needs nvcc)")
                handle = ctypes.CDLL(_LIB_PATH)
                for name, (res, args) in SIGNATURES.items():
                    fn = getattr(handle, name)
                    fn.restype = res
                    fn.argtypes = args
                _lib = handle
    return _lib


def status_string(code: int) -> str:
    return lib().fa2_status_string(int(code)).decode()


def check(code: int) -> None:
    if code != FA2_OK:
        raise FA2Error(code)


def last_device_status() -> int:
    return int(lib().fa2_last_device_status())


def clear_device_status() -> None:
    check(lib().fa2_clear_device_status())
