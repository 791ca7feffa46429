"""ctypes handle on libfa.so (the CUDA kernels behind the C ABI in include/fa.h).

The library must have been built (``python -m exact_attention_159_b200.build``
or ``__graft_entry__.build()``); nothing here falls back to another
implementation when it is missing.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

_lock = threading.Lock()
_lib = None

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(6)

# Every entry point declared in include/fa.h: name -> (restype, argtypes)
_P = ctypes.c_void_p
_I = ctypes.c_int
SIGNATURES = {
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, ctypes.c_float, _I, _P]),
    "fa_bwd_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "fa_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _I,
                    ctypes.c_float, _I, _P]),
    "fa_fwd_qk": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, _P]),
    "fa_bwd_qk_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "fa_bwd_qk": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _I, _I, _I,
                       ctypes.c_float, _I, _P]),
    "fa_fwd_accumulate": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, _I, _P]),
    "fa_bwd_prepare": (_I, [_P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _I, _P]),
    "fa_bwd_accumulate": (_I, [_P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P, _I, _I, _I, _I, _I, _I,
                               ctypes.c_float, _I, _I, _P]),
    "fa_bwd_finish": (_I, [_P, ctypes.c_size_t, _P, _I, _I, _I, _I, ctypes.c_float, _P]),
    "fa_lse_merge": (_I, [_P, _P, _P, _P, ctypes.c_int64, _I, _I, _P]),
    "fa_accumulate_bf16": (_I, [_P, _P, ctypes.c_int64, _I, _P]),
    "fa_accumulate_f32": (_I, [_P, _P, ctypes.c_int64, _P]),
    "fa_convert_f32_bf16": (_I, [_P, _P, ctypes.c_int64, _P]),
    "fa_strerror": (ctypes.c_char_p, [_I]),
    "fa_last_device_status": (_I, [_P, ctypes.POINTER(ctypes.c_int)]),
    "fa_set_softmax_options": (_I, [ctypes.c_float, _I]),
    "fa_exp2_eval": (_I, [_P, _P, ctypes.c_int64, _I, _P]),
    "fa_profile_next": (_I, [_I, _P, _P]),
    "fa_bwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, ctypes.c_float, _I, _P]),
    "fa_selftest_wait_timeout": (_I, [_P]),
    "fa_sm_clock_probe": (_I, [_P, _P]),
    "fa_set_forward_variant": (_I, [_I]),
    "fa_set_backward_variant": (_I, [_I]),
    "fa_version": (_I, []),
}


class FAError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {lib().fa_strerror(code).decode()} (status {code})")


def lib_path() -> str:
    return _build.LIB


def lib():
    """Load libfa.so once; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            path = lib_path()
            if not os.path.exists(path):
                raise ImportError(f"libfa.so not built ({path}); run exact_attention_159_b200.build.build()")
            handle = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(handle, name)
                fn.restype = res
                fn.argtypes = args
            _lib = handle
        return _lib


def check(code: int, what: str) -> None:
    if code != FA_OK:
        raise FAError(code, what)
