"""ctypes binding over libattn_blocks.so (include/attn_blocks.h): the
building-block checks.  Same names and arguments as the C functions."""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn_blocks.so")
_lock = threading.Lock()
_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build with "
                                  "`python -m exact_attention_152_b200.build`")
            l = ctypes.CDLL(LIB_PATH)
            for name, args in (("blocks_mma_ss", [_P, _P, _P, _I, _P]),
                               ("blocks_mma_ts", [_P, _P, _P, _I, _P]),
                               ("blocks_swizzle_roundtrip", [_P, _P, _P, _I, _P]),
                               ("blocks_exp2", [_P, _P, _P, _I, _P]),
                               ("blocks_mma_e4m3_ss", [_P, _P, _P, _P]),
                               ("blocks_mma_e4m3_ts", [_P, _P, _P, _P]),
                               ("blocks_pack_e4m3", [_P, _P, _I, _P]),
                               ("blocks_status_sync", [_P])):
                f = getattr(l, name)
                f.argtypes = args
                f.restype = _I
            _lib = l
    return _lib


def blocks_mma_ss(a, b, c, d, stream) -> int:
    return lib().blocks_mma_ss(a, b, c, d, stream)


def blocks_mma_ts(p, v, c, d, stream) -> int:
    return lib().blocks_mma_ts(p, v, c, d, stream)


def blocks_swizzle_roundtrip(x, y_tma, y_plain, d, stream) -> int:
    return lib().blocks_swizzle_roundtrip(x, y_tma, y_plain, d, stream)


def blocks_exp2(x, y_mufu, y_poly, n, stream) -> int:
    return lib().blocks_exp2(x, y_mufu, y_poly, n, stream)


def blocks_mma_e4m3_ss(a, b, c, stream) -> int:
    return lib().blocks_mma_e4m3_ss(a, b, c, stream)


def blocks_mma_e4m3_ts(p, v, c, stream) -> int:
    return lib().blocks_mma_e4m3_ts(p, v, c, stream)


def blocks_pack_e4m3(x, y, n4, stream) -> int:
    return lib().blocks_pack_e4m3(x, y, n4, stream)


def blocks_status_sync(stream) -> int:
    return lib().blocks_status_sync(stream)
