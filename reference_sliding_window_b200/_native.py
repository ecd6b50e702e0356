"""ctypes loader for librswa.so: one Python callable per C entry point of
include/rswa.h, with argument types declared.  Loading fails loudly if the
library has not been built; there is no other implementation to fall back on.
"""

from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librswa.so")

# rswa_status
OK, ERR_ARG, ERR_STATE, ERR_CAPACITY, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE = range(7)
STATUS_NAMES = ["RSWA_OK", "RSWA_ERR_ARG", "RSWA_ERR_STATE", "RSWA_ERR_CAPACITY",
                "RSWA_ERR_UNSUPPORTED", "RSWA_ERR_CUDA", "RSWA_ERR_DEVICE"]
# rswa_dtype / rswa_mode / rswa_forward_flags
F32, BF16 = 0, 1
MODE_RSWA, MODE_FULL = 0, 1
FLAG_BIDIR_PREFIX = 1

_i, _f, _p, _sz = C.c_int, C.c_float, C.c_void_p, C.c_size_t
_PROTOS = {
    "rswa_cache_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "rswa_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "rswa_init": (_i, [C.POINTER(_p), _i, _i, _i, _i, _i, _i, _i, _i, _p, _p, _p, _sz, _p]),
    "rswa_load_reference": (_i, [_p, _p, _p, _i, C.POINTER(C.c_int32)]),
    "rswa_load_packed": (_i, [_p, _p, _p, _i, C.POINTER(C.c_int32), _i]),
    "rswa_load_reference_chunk": (_i, [_p, _p, _p, _i, C.POINTER(C.c_int32)]),
    "rswa_append": (_i, [_p, _p, _p]),
    "rswa_decode": (_i, [_p, _p, _p, _f]),
    "rswa_append_decode": (_i, [_p, _p, _p, _p, _p, _f]),
    "rswa_append_decode_layers": (_i, [C.POINTER(_p), _i, C.POINTER(_p), C.POINTER(_p), C.POINTER(_p),
                                      C.POINTER(_p), _f]),
    "rswa_cache_len": (_i, [_p, C.POINTER(C.c_int32)]),
    "rswa_step_count": (_i, [_p, C.POINTER(C.c_int32)]),
    "rswa_cache_positions": (_i, [_p, _i, C.POINTER(C.c_int64), _i, C.POINTER(_i)]),
    "rswa_reset": (_i, [_p]),
    "rswa_set_stream": (_i, [_p, _p]),
    "rswa_check": (_i, [_p]),
    "rswa_destroy": (None, [_p]),
    "rswa_masked_forward": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _p]),
    "rswa_masked_forward_ex": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _i, _p]),
    "rswa_masked_forward_fill": (_i, [_p, _p, _p, _p, _p, _i, _i, _f, _i]),
    "rswa_masked_forward_varlen": (_i, [_p, _p, _p, _p, C.POINTER(C.c_int32), C.POINTER(C.c_int32), _i, _i,
                                       _i, _i, _i, _f, _i, _p]),
    "rswa_decode_noalloc": (_i, [_p, _p, _i, C.POINTER(C.c_int32), _p, _p, _i, _i, _i, _i, _f, _p]),
    "rswa_decode_noalloc_check": (_i, [_p]),
    "rswa_plan_decode": (_i, [_i, _i, C.POINTER(C.c_int32), _i, _i, _i, _i, C.POINTER(C.c_int32), _i,
                              C.POINTER(C.c_int32), _i, C.POINTER(_i), C.POINTER(_i), C.POINTER(_i)]),
    "rswa_last_error": (C.c_char_p, []),
    "rswa_version": (C.c_char_p, []),
}

_lib = None


class RSWAError(RuntimeError):
    def __init__(self, status: int, message: str):
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else str(status)
        super().__init__(f"{name}: {message}")
        self.status = status


def lib() -> C.CDLL:
    """The loaded library (loaded on first use)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m reference_sliding_window_b200.build` "
                "(or __graft_entry__.build()); the library has no non-CUDA implementation")
        handle = C.CDLL(LIB_PATH)
        for name, (res, args) in _PROTOS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def check(status: int) -> None:
    if status != OK:
        raise RSWAError(status, lib().rswa_last_error().decode())
