"""ctypes loader for libfa_b200.so: the symbol table of include/fa.h.

There is no fallback: if the library is missing the call fails loudly."""
from __future__ import annotations

import ctypes
import os
import threading

from .build import LIB

_lock = threading.Lock()
_handle = None

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(5)

# name -> (restype, argtypes), exactly the declarations of include/fa.h
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_u32, _u64 = ctypes.c_uint32, ctypes.c_uint64
SIGNATURES = {
    "fa_forward": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp]),
    "fa_backward_workspace_size": (_sz, [_i, _i, _i, _i]),
    "fa_backward": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                         _i, _i, _i, _i, _f, _i, _vp, _sz, _vp]),
    "fa_backward_preprocess": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _sz, _vp]),
    "fa_backward_main": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _sz,
                              _vp]),
    "fa_backward_dq_convert": (_i, [_vp, _i, _i, _i, _i, _f, _vp, _sz, _vp]),
    "fa_backward_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _i, _i, _i, _i, _f, _i, _vp]),
    "fa_forward_f16": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp]),
    "fa_backward_f16": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                             _i, _i, _i, _i, _f, _i, _vp, _sz, _vp]),
    "fa_forward_masked": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _i, _vp,
                               _vp]),
    "fa_backward_masked": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _i, _i, _i, _i, _f, _i, _i, _i, _vp, _vp, _sz, _vp]),
    "fa_dropout_rate": (_f, [_f]),
    "fa_launch_plan": (_i, [_i, _i, _i, _i, _i, _vp, _vp, _vp]),
    "fa_forward_dropout": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _i, _vp,
                                _f, _u64, _u32, _vp]),
    "fa_backward_dropout": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _i, _i, _i, _i, _f, _i, _i, _i, _vp, _f, _u64, _u32,
                                 _vp, _sz, _vp]),
    "fa_forward_dropout_heads": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _i,
                                      _vp, _f, _u64, _u32, _i, _vp]),
    "fa_backward_dropout_heads": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                       _i, _i, _i, _i, _f, _i, _i, _i, _vp, _f, _u64, _u32,
                                       _i, _vp, _sz, _vp]),
    "fa_forward_f32": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp]),
    "fa_backward_f32": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                             _i, _i, _i, _i, _f, _i, _vp, _sz, _vp]),
    "fa_get_status": (_i, [_vp]),
    "fa_watchdog_selftest": (_i, [_i, _vp]),
    "fa_status_string": (ctypes.c_char_p, [_i]),
    "fa_version": (ctypes.c_char_p, []),
}


class FAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """The loaded library. Raises if libfa_b200.so has not been built."""
    global _handle
    with _lock:
        if _handle is None:
            if not os.path.exists(LIB):
                raise RuntimeError(
                    f"{LIB} is missing: build it with "
                    "`python -m io_aware_attention_flashattention_b200.build`")
            h = ctypes.CDLL(LIB)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(h, name)
                fn.restype = res
                fn.argtypes = args
            _handle = h
    return _handle


def status_string(status: int) -> str:
    return lib().fa_status_string(int(status)).decode()


def check(fn: str, status: int) -> None:
    if status != FA_OK:
        raise FAError(fn, status)
