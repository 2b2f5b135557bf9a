"""ctypes binding of libfa.so (the C ABI declared in include/fa.h).

Argument marshalling only: every step of the attention path runs in the
library's CUDA kernels.  Importing this module fails loudly when the library
has not been built; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_OK = 0
STATUS_NAMES = {
    0: "FA_OK",
    1: "FA_ERR_INVALID_ARG",
    2: "FA_ERR_UNSUPPORTED",
    3: "FA_ERR_ALIGNMENT",
    4: "FA_ERR_ARCH",
    5: "FA_ERR_LAUNCH",
    6: "FA_ERR_DEVICE_TIMEOUT",
    7: "FA_ERR_WORKSPACE",
    8: "FA_ERR_SCRATCH_LIMIT",
}
STATUS_CODES = {v: k for k, v in STATUS_NAMES.items()}


class FAError(RuntimeError):
    """A call into libfa.so returned a non-zero fa_status."""

    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python exact_io_aware_55_b200/build.py` "
            "(the CUDA library is required; there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_fwd.restype = i
    lib.fa_fwd_fp8.argtypes = [vp, vp, vp, f, f, f, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_fwd_fp8.restype = i
    lib.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    lib.fa_bwd_workspace_size.restype = sz
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp]
    lib.fa_bwd.restype = i
    lib.fa_fwd_decode.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, sz, vp]
    lib.fa_fwd_decode.restype = i
    lib.fa_fwd_decode_workspace_size.argtypes = [i, i, i, i, i]
    lib.fa_fwd_decode_workspace_size.restype = sz
    lib.fa_fwd_standard.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp]
    lib.fa_fwd_standard.restype = i
    lib.fa_fwd_standard_workspace_size.argtypes = [i, i, i, i]
    lib.fa_fwd_standard_workspace_size.restype = sz
    lib.fa_bwd_fp8.argtypes = [vp, vp, vp, f, f, f, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp]
    lib.fa_bwd_fp8.restype = i
    lib.fa_bwd_fp8_workspace_size.argtypes = [i, i, i, i]
    lib.fa_bwd_fp8_workspace_size.restype = sz
    lib.fa_bwd_events.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz,
                                  ctypes.POINTER(vp), vp]
    lib.fa_bwd_events.restype = i
    lib.fa_fwd_plan.argtypes = [i, i, i, i, i, ctypes.POINTER(i), ctypes.POINTER(i), ctypes.POINTER(i)]
    lib.fa_fwd_plan.restype = i
    lib.fa_get_device_status.argtypes = [vp]
    lib.fa_get_device_status.restype = i
    lib.fa_bwd_deterministic.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp]
    lib.fa_bwd_deterministic.restype = i
    lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_bwd_noalloc.restype = i
    lib.fa_bwd_noalloc_max_bytes.argtypes = []
    lib.fa_bwd_noalloc_max_bytes.restype = sz
    lib.fa_strerror.argtypes = [i]
    lib.fa_strerror.restype = ctypes.c_char_p
    lib.fa_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.fa_device_status.restype = i
    lib.fa_watchdog_selftest.argtypes = [ctypes.c_uint32, vp]
    lib.fa_watchdog_selftest.restype = i
    lib.fa_version.argtypes = []
    lib.fa_version.restype = i
    return lib


lib = _load()


def check(status: int) -> None:
    if status != FA_OK:
        raise FAError(status, lib.fa_strerror(status).decode())


def strerror(status: int) -> str:
    return lib.fa_strerror(status).decode()
