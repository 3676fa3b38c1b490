"""ctypes loader for libgqa_attn.so (the C ABI declared in include/gqa_attn.h).

The library is built in-tree by ``long_context_causal_flash_b200.build``.  There is
no fallback: if the shared library is missing, every call raises.  With
GQA_ATTN_DEBUG_BOUNDS=1 in the environment the checked build
(libgqa_attn_debug_bounds.so, ``build --debug-bounds``) is loaded instead.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(
    HERE, "libgqa_attn_debug_bounds.so" if os.environ.get("GQA_ATTN_DEBUG_BOUNDS") == "1" else "libgqa_attn.so")

GQA_F32, GQA_BF16, GQA_F32_TC = 0, 1, 2
GQA_MASK_CAUSAL, GQA_MASK_PREFIX_BRANCH = 0, 1
GQA_OK = 0
GQA_ERR_INVALID_ARG = -1
GQA_ERR_UNSUPPORTED = -2
GQA_ERR_MISALIGNED = -3
GQA_ERR_WORKSPACE = -4
GQA_ERR_LAUNCH = -5
GQA_ERR_DEVICE_TIMEOUT = -6
GQA_ERR_DEVICE_BOUNDS = -7

# name -> (restype, argtypes), mirroring include/gqa_attn.h
_c = ctypes
SIGNATURES = {
    "gqa_attn_workspace_bytes": (_c.c_size_t, [_c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64,
                                               _c.c_int, _c.c_int, _c.c_int, _c.c_int]),
    "gqa_attn_fwd": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                _c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int, _c.c_int,
                                _c.c_int, _c.c_int64, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_size_t,
                                _c.c_void_p]),
    "gqa_attn_split_hint": (_c.c_int, [_c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int,
                                       _c.c_int, _c.c_int]),
    "gqa_attn_split_workspace_bytes": (_c.c_size_t, [_c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64,
                                                     _c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_int]),
    "gqa_attn_fwd_split": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                      _c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int, _c.c_int,
                                      _c.c_int, _c.c_int64, _c.c_void_p, _c.c_void_p, _c.c_int, _c.c_void_p,
                                      _c.c_size_t, _c.c_void_p]),
    "gqa_attn_bwd_workspace_bytes": (_c.c_size_t, [_c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64,
                                                   _c.c_int, _c.c_int, _c.c_int, _c.c_int]),
    "gqa_attn_bwd": (_c.c_int, [_c.c_void_p] * 9 + [_c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int,
                                                    _c.c_int, _c.c_int, _c.c_int64, _c.c_void_p, _c.c_void_p,
                                                    _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "gqa_attn_bwd_offset": (_c.c_int, [_c.c_void_p] * 9 + [_c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64,
                                                           _c.c_int, _c.c_int, _c.c_int64, _c.c_void_p, _c.c_size_t,
                                                           _c.c_void_p]),
    "gqa_attn_tile_sizes": (_c.c_int, [_c.c_int, _c.c_int, _c.c_int, _c.POINTER(_c.c_int),
                                       _c.POINTER(_c.c_int)]),
    "gqa_attn_tile_plan": (_c.c_int, [_c.c_int, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int, _c.c_int,
                                      _c.c_int64, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_size_t,
                                      _c.c_void_p, _c.c_void_p, _c.c_void_p]),
    "gqa_attn_fwd_static_ws": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                          _c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int,
                                          _c.c_int, _c.c_int, _c.c_int64, _c.c_void_p, _c.c_void_p,
                                          _c.c_void_p]),
    "gqa_attn_fwd_offset": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                       _c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int, _c.c_int,
                                       _c.c_int64, _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "gqa_attn_merge": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                  _c.c_int64, _c.c_int, _c.c_int, _c.c_int, _c.c_void_p]),
    "gqa_attn_status": (_c.c_int, [_c.c_void_p, _c.c_void_p]),
    "gqa_attn_selftest_wait": (_c.c_int, [_c.c_void_p, _c.c_size_t, _c.c_int64, _c.c_void_p]),
    "gqa_attn_selftest_bounds": (_c.c_int, [_c.c_void_p, _c.c_size_t, _c.c_int, _c.c_void_p]),
    "gqa_attn_probe_ffma2": (_c.c_int, [_c.c_void_p, _c.c_int, _c.c_int, _c.c_int, _c.c_void_p]),
    "gqa_attn_strerror": (_c.c_char_p, [_c.c_int]),
}

_lib = None


class GqaAttnError(RuntimeError):
    """A nonzero status from libgqa_attn."""

    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status} ({strerror(status)})")


def load() -> ctypes.CDLL:
    """The loaded library, with argument types set.  Raises if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m long_context_causal_flash_b200.build` "
                "(there is no non-CUDA fallback)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def strerror(status: int) -> str:
    if _lib is None and not os.path.exists(LIB_PATH):
        return "unknown (library not built)"
    return load().gqa_attn_strerror(int(status)).decode()


def check(fn: str, status: int) -> None:
    if status != GQA_OK:
        raise GqaAttnError(fn, status)
