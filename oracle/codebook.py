"""Oracle: lossless codebook codec (table of unique values + packed indices).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Follows "Codebook Lossless Compression: когда 25% памяти значат больше, чем
кажется" (ai-manual.ru), section "Как работает эта магия? (Коротко, без
формул)": the weights become a dictionary plus a list of indices, and at
inference the original values are substituted back with no approximation;
and "無損 LLM 壓縮減少 10-25% RAM" (setupai.cc), key points and "技術深入":
indices into the unique weights are bit-packed (12-13 bits on the models it
reports).

Readings where the pages are silent: the dictionary is every distinct 16-bit
pattern of the tensor in ascending order (the pages' "clusters of similar
values" and K-means variants are the lossy modes and are not built); the
index width is the smallest k with 2^k >= U (k = 0 for a one-entry table);
indices are packed least significant bit first.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import blob as B
from ._native import lib, ptr


def index_bits(U: int) -> int:
    """Smallest k >= 0 with 2**k >= U."""
    k = 0
    while (1 << k) < U:
        k += 1
    return k


def encode(w: np.ndarray) -> np.ndarray:
    """Compress BF16 bit patterns into a codebook blob (uint8 array)."""
    w = np.ascontiguousarray(w, dtype=np.uint16).reshape(-1)
    n = w.size
    table = np.unique(w)                       # ascending distinct patterns
    U = int(table.size)
    k = index_bits(U)
    idx = np.searchsorted(table, w).astype(np.uint32)
    packed_bytes = B.align(-(-n * k // 8) + 16, 16) if k else 0
    words = np.zeros(packed_bytes // 4, np.uint32)
    if k:
        lib().orc_pack_lsb(ptr(idx, ctypes.c_uint32), n, k, ptr(words, ctypes.c_uint32))
    header = dict(magic=B.MAGIC, version=B.VERSION, codec=B.CODEC_CODEBOOK, n=n,
                  header_bytes=B.HEADER_BYTES, flags=0, U=U, k=k, packed_bytes=packed_bytes)
    return B.assemble(header, [("table", table.astype(np.uint16)), ("packed", words)])


def _parts(blob: np.ndarray, h: dict):
    if h["k"] > 16 or h["U"] > 65536 or (h["n"] and h["U"] == 0) or (1 << h["k"]) < h["U"]:
        raise ValueError("bad codebook parameters")
    if h["k"] and h["packed_bytes"] * 8 < h["n"] * h["k"]:
        raise ValueError("packed section too short")
    table = B.section(blob, h["off_table"], 2 * h["U"], np.uint16)
    words = B.section(blob, h["off_packed"], h["packed_bytes"] // 4 * 4, np.uint32)
    return table, words


def decode_range(blob: np.ndarray, i0: int, count: int) -> np.ndarray:
    """Weights [i0, i0 + count) of a codebook blob, each read on its own."""
    blob = np.asarray(blob, np.uint8)
    h = B.unpack_header(blob)
    if h["codec"] != B.CODEC_CODEBOOK:
        raise ValueError("not a codebook blob")
    if i0 < 0 or i0 + count > h["n"]:
        raise ValueError("range outside the tensor")
    table, words = _parts(blob, h)
    out = np.empty(count, np.uint16)
    if h["k"] == 0:
        out[:] = table[0] if count else 0
        return out
    rc = lib().orc_cb_decode(ptr(words, ctypes.c_uint32), i0, count, h["k"],
                             ptr(table, ctypes.c_uint16), h["U"], ptr(out, ctypes.c_uint16))
    if rc != 0:
        raise ValueError("index outside the table")
    return out


def decode(blob: np.ndarray) -> np.ndarray:
    h = B.unpack_header(np.asarray(blob, np.uint8))
    return decode_range(blob, 0, h["n"])


def bits_per_weight(blob: np.ndarray) -> float:
    h = B.unpack_header(blob)
    return 8.0 * h["total_bytes"] / max(1, h["n"])
