"""ctypes declarations of libmuon_b200.so (the C ABI declared in include/muon.h).

The library is loaded lazily on first use and NEVER replaced by anything else:
if it cannot be loaded the caller gets an ImportError naming the file, and on
a machine without the sm_100a device every compute call returns
MUON_ERR_UNSUPPORTED / MUON_ERR_CUDA as an exception.  There is no CPU path.
"""
from __future__ import annotations

import ctypes
import os
import threading

#: The in-tree build; MUON_B200_LIB may name another build of the same
#: sources (e.g. a variant compiled with different tile parameters).
LIB_PATH = os.environ.get("MUON_B200_LIB") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "libmuon_b200.so")

MUON_BF16 = 0
MUON_FP32 = 1
MUON_CAUTIOUS_WD = 1

STATUS_NAMES = {
    0: "MUON_OK",
    -1: "MUON_ERR_ARG",
    -2: "MUON_ERR_SHAPE",
    -3: "MUON_ERR_CUDA",
    -4: "MUON_ERR_ALLOC",
    -5: "MUON_ERR_DEVICE_TIMEOUT",
    -6: "MUON_ERR_UNSUPPORTED",
}

_P = ctypes.c_void_p
_PP = ctypes.POINTER(ctypes.c_void_p)
_I = ctypes.c_int
_F = ctypes.c_float
_I64P = ctypes.POINTER(ctypes.c_int64)

#: name -> (restype, argtypes); every entry point of include/muon.h.
SIGNATURES = {
    "muon_ns_orthogonalize": (_I, [_I, _I, _I, _PP, _F, _F, _F, _I, _I, _P]),
    "muon_ns_orthogonalize_static": (_I, [_I, _I, _I, _PP, _F, _F, _F, _I, _P, _P]),
    "muon_ns_orthogonalize_schedule": (_I, [_I, _I, _I, _PP, ctypes.POINTER(_F), _I, _I, _P]),
    "muon_step": (_I, [_I, _PP, _PP, _PP, _I64P, _F, _I, _F, _F, _I, _P]),
    "muon_step_ex": (_I, [_I, _PP, _PP, _PP, _I64P, _F, _I, _F, _F, _I, ctypes.POINTER(_F), _I, _PP, _F, _P]),
    "muon_momentum": (_I, [_I, _PP, _PP, _I64P, _F, _I, _P, _P]),
    "muon_apply": (_I, [_I, _PP, _PP, _I64P, _F, _F, _P]),
    "muon_apply_ex": (_I, [_I, _PP, _PP, _I64P, _F, _F, _I, _PP, _P]),
    "muon_gram_bf16": (_I, [_I, _I, _I, _P, _P, _P]),
    "muon_poly_bf16": (_I, [_I, _I, _P, _P, _F, _F, _P]),
    "muon_bx_bf16": (_I, [_I, _I, _I, _P, _P, _P, _P, _F, _P]),
    "muon_bx_apply_bf16": (_I, [_I, _I, _I, _I, _P, _I, _P, _P, _PP, _I, _F, _F, _F, _I, _P]),
    "muon_get_status": (_I, [_P]),
    "muon_last_error": (ctypes.c_char_p, []),
    "muon_release": (_I, []),
    "muon_workspace_bytes": (_I, [_P, ctypes.POINTER(ctypes.c_longlong)]),
    "muon_set_wait_timeout_ms": (_I, [_I]),
    "muon_set_fault_injection": (_I, [_I]),
    "muon_profile_begin": (_I, []),
    "muon_profile_end": (_I, [_I, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)]),
    "muon_version": (_I, []),
}

#: muon_kernel_kind names, in enum order.
KERNEL_KINDS = ["flat", "cast", "gram", "poly", "bx", "out", "simt", "sums", "prep", "scale", "bx_apply",
                "norm"]

_lock = threading.Lock()
_lib = None


class MuonError(RuntimeError):
    """A negative muon_status returned by the library."""

    def __init__(self, code, message):
        self.code = code
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {message}")


def lib():
    """The loaded library (loaded once; raises ImportError if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is not built; run `python -m newton_schulz_12_b200.build` "
                    "(the library has no fallback implementation)")
            handle = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(handle, name)
                fn.restype = res
                fn.argtypes = args
            _lib = handle
    return _lib


def check(rc):
    if rc != 0:
        msg = lib().muon_last_error()
        raise MuonError(rc, msg.decode() if msg else "")
    return rc


def ptr_array(ptrs):
    arr = (ctypes.c_void_p * max(1, len(ptrs)))()
    for i, p in enumerate(ptrs):
        arr[i] = p
    return arr


def shape_array(shapes):
    arr = (ctypes.c_int64 * max(1, 2 * len(shapes)))()
    for i, (r, c) in enumerate(shapes):
        arr[2 * i] = r
        arr[2 * i + 1] = c
    return arr
