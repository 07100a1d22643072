"""Oracle: builds and loads ``native.c`` (plain C, gcc -O2) with ctypes.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "native.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile native.c into oracle/_build/liboracle.so if it is missing or stale."""
    with _lock:
        if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
            os.makedirs(_BUILD, exist_ok=True)
            tmp = _SO + f".{os.getpid()}.tmp"
            subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC],
                           check=True)
            os.replace(tmp, _SO)
    return _SO


_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_u64p = ctypes.POINTER(ctypes.c_uint64)
_u64 = ctypes.c_uint64


def lib():
    global _lib
    if _lib is None:
        so = build()
        L = ctypes.CDLL(so)
        L.orc_split.argtypes = [_u16p, _u64, _u8p, _u8p]
        L.orc_merge.argtypes = [_u8p, _u8p, _u64, _u16p]
        L.orc_histogram.argtypes = [_u8p, _u64, _u64p]
        L.orc_df11_emit.argtypes = [_u8p, _u64, _u8p, _u32p, _u32p]
        L.orc_df11_emit.restype = _u64
        L.orc_df11_decode_syms.argtypes = [_u32p, _u64, _u64, _u64, _u32p, _u32p, _u32p, _u8p,
                                           ctypes.c_int, _u8p, _u8p, _u64p]
        L.orc_df11_decode_syms.restype = ctypes.c_int
        L.orc_pack_lsb.argtypes = [_u32p, _u64, ctypes.c_uint32, _u32p]
        L.orc_cb_decode.argtypes = [_u32p, _u64, _u64, ctypes.c_uint32, _u16p, ctypes.c_uint32, _u16p]
        L.orc_cb_decode.restype = ctypes.c_int
        _lib = L
    return _lib


def ptr(a: np.ndarray | None, ctype):
    if a is None:
        return ctypes.cast(None, ctypes.POINTER(ctype))
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))
