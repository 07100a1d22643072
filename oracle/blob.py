"""Oracle: the compressed-blob container (header + sections).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages fix no file format; this is the repository's own container, written
here independently of the library's C implementation of the same layout.
All integers little-endian. The header is 256 bytes; every section starts at
a multiple of 16 bytes (this writer uses 256) inside ``total_bytes``.
"""
from __future__ import annotations

import struct

import numpy as np

MAGIC = 0x3143574C            # bytes "LWC1"
VERSION = 1
CODEC_DFLOAT11 = 1
CODEC_CODEBOOK = 2
FLAG_SINGLE_EXPONENT = 1
FLAG_CHUNK_COUNTS = 2         # DFloat11: a u8 code count per chunk is stored ("counts")
ELEM_BF16 = 0   # DFloat11 element types (header field "elem")
ELEM_FP32 = 1
ELEM_FP16 = 2
HEADER_BYTES = 256
SECTION_ALIGN = 256

# (field, byte offset, struct code)
COMMON = (
    ("magic", 0, "I"), ("version", 4, "H"), ("codec", 6, "H"), ("n", 8, "Q"),
    ("total_bytes", 16, "Q"), ("header_bytes", 24, "I"), ("flags", 28, "I"),
)
DF11 = (
    ("chunk_bytes", 32, "I"), ("threads_per_block", 36, "I"), ("max_len", 40, "I"),
    ("n_tables", 44, "I"), ("n_chunks", 48, "Q"), ("n_blocks", 56, "Q"),
    ("total_bits", 64, "Q"), ("max_block_count", 72, "I"), ("const_exp", 76, "I"),
    ("off_lengths", 80, "Q"), ("off_lut", 88, "Q"), ("off_gaps", 96, "Q"),
    ("off_blkoff", 104, "Q"), ("off_stream", 112, "Q"), ("stream_bytes", 120, "Q"),
    ("off_sm", 128, "Q"), ("elem", 136, "I"), ("off_lo", 144, "Q"), ("lo_bytes", 152, "Q"),
    ("off_counts", 160, "Q"),
)
CODEBOOK = (
    ("U", 32, "I"), ("k", 36, "I"), ("off_table", 40, "Q"), ("off_packed", 48, "Q"),
    ("packed_bytes", 56, "Q"),
)


def _fields(codec):
    return COMMON + (DF11 if codec == CODEC_DFLOAT11 else CODEBOOK)


def pack_header(h: dict) -> bytes:
    buf = bytearray(HEADER_BYTES)
    for name, off, code in _fields(h["codec"]):
        struct.pack_into("<" + code, buf, off, int(h.get(name, 0)))
    return bytes(buf)


def unpack_header(blob) -> dict:
    raw = bytes(np.asarray(blob, dtype=np.uint8)[:HEADER_BYTES])
    if len(raw) < HEADER_BYTES:
        raise ValueError("blob shorter than its header")
    codec = struct.unpack_from("<H", raw, 6)[0]
    if codec not in (CODEC_DFLOAT11, CODEC_CODEBOOK):
        raise ValueError(f"unknown codec {codec}")
    h = {name: struct.unpack_from("<" + code, raw, off)[0] for name, off, code in _fields(codec)}
    if h["magic"] != MAGIC or h["version"] != VERSION or h["header_bytes"] != HEADER_BYTES:
        raise ValueError("bad magic/version/header size")
    return h


def align(x: int, a: int = SECTION_ALIGN) -> int:
    return (x + a - 1) // a * a


def assemble(header: dict, sections: list[tuple[str, np.ndarray]]) -> np.ndarray:
    """Lay the sections out after the header (each at a 256-byte boundary),
    record their offsets as header['off_<name>'], and return the blob bytes."""
    pos = HEADER_BYTES
    placed = []
    for name, arr in sections:
        data = np.ascontiguousarray(arr).view(np.uint8).reshape(-1)
        pos = align(pos)
        header["off_" + name] = pos
        placed.append((pos, data))
        pos += data.size
    total = align(pos, 16)
    header["total_bytes"] = total
    blob = np.zeros(total, dtype=np.uint8)
    blob[:HEADER_BYTES] = np.frombuffer(pack_header(header), dtype=np.uint8)
    for off, data in placed:
        blob[off:off + data.size] = data
    return blob


def section(blob: np.ndarray, off: int, nbytes: int, dtype=np.uint8) -> np.ndarray:
    if off % 16 or off + nbytes > blob.size:
        raise ValueError("section misaligned or outside the blob")
    out = np.empty(nbytes // np.dtype(dtype).itemsize, dtype=dtype)
    out.view(np.uint8)[:] = blob[off:off + out.nbytes]
    return out
