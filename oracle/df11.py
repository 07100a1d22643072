"""Oracle: DFloat11-style codec (Huffman-coded exponent + raw sign|mantissa byte).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Follows "Koniec z kompromisami! DFloat11 ratuje dokładność modeli AI ..."
(gadzety360.pl):

* section "Przełom: DFloat11 – bezstratna kompresja z wydajnością GPU":
  BF16 = 1 sign + 8 exponent + 7 mantissa bits; the exponent carries about
  2.6 bits of information; it alone is Huffman coded, sign and mantissa are
  untouched; the result is about 70 % of the BF16 size (about 11 bits per
  weight) and decodes bit for bit to the original.
* section "Jak to działa w praktyce? Magia na poziomie GPU": Huffman
  decoding is sequential; the GPU decoder uses small linked lookup tables and
  two phases in which threads first count what they will decode and then,
  after a synchronisation, write it at the right place. For that the blob
  carries, per fixed-size chunk of the bitstream, the offset of the first code
  that starts in it (``gaps``) and, per block of chunks, the index of the first
  weight it decodes (``blkoff``).

Encoding steps, in the order the pages give them: split each weight into its
exponent and its sign|mantissa byte; count exponents; build the Huffman code
(``oracle.huffman``); write the codes one after another; record the chunk and
block offsets. Decoding is the plain sequential reading of that bitstream,
one bit at a time, and the merge of each exponent with its sign|mantissa byte.
"""
from __future__ import annotations

import numpy as np

from . import blob as B
from . import huffman as H
from ._native import lib, ptr

import ctypes

DEFAULT_CHUNK_BYTES = 36
DEFAULT_THREADS_PER_BLOCK = 256
DEFAULT_MAX_LEN = 32
FORMAT_MAX_LEN = 32


def split(w: np.ndarray):
    """Exponent byte and sign|mantissa byte of every BF16 pattern."""
    w = np.ascontiguousarray(w, dtype=np.uint16).reshape(-1)
    e = np.empty(w.size, np.uint8)
    s = np.empty(w.size, np.uint8)
    lib().orc_split(ptr(w, ctypes.c_uint16), w.size, ptr(e, ctypes.c_uint8), ptr(s, ctypes.c_uint8))
    return e, s


def merge(e: np.ndarray, s: np.ndarray) -> np.ndarray:
    w = np.empty(e.size, np.uint16)
    lib().orc_merge(ptr(e, ctypes.c_uint8), ptr(s, ctypes.c_uint8), e.size, ptr(w, ctypes.c_uint16))
    return w


def histogram(e: np.ndarray) -> np.ndarray:
    counts = np.zeros(256, np.uint64)
    lib().orc_histogram(ptr(e, ctypes.c_uint8), e.size, ptr(counts, ctypes.c_uint64))
    return counts


def code_for(w: np.ndarray, max_len: int = DEFAULT_MAX_LEN):
    """(counts, lengths, codes) of the exponent code of a tensor."""
    e, _ = split(w)
    counts = histogram(e)
    lengths = H.limited_lengths(counts, max_len)
    return counts, lengths, H.canonical_codes(lengths)


def chunk_index(code_lengths_per_weight: np.ndarray, total_bits: int, chunk_bits: int,
                threads_per_block: int):
    """gaps[c] and blkoff[b] from the code start positions.

    starts[i] = bit where code i starts (exclusive prefix sum of the code
    lengths), with starts[n] = total_bits. For chunk c starting at bit
    c*chunk_bits < total_bits, gaps[c] = (first start >= c*chunk_bits) -
    c*chunk_bits; chunks at or beyond total_bits get 0. blkoff[b] = number of
    codes that start before the first bit of block b; blkoff[last] = n.
    """
    n = code_lengths_per_weight.size
    starts = np.zeros(n + 1, np.uint64)
    np.cumsum(code_lengths_per_weight, dtype=np.uint64, out=starts[1:])
    assert int(starts[-1]) == total_bits
    n_chunks = -(-total_bits // chunk_bits)
    n_blocks = -(-n_chunks // threads_per_block)
    gaps = np.zeros(n_blocks * threads_per_block, np.uint8)
    chunk_starts = np.arange(n_chunks, dtype=np.uint64) * np.uint64(chunk_bits)
    j = np.searchsorted(starts, chunk_starts, side="left")
    g = starts[j] - chunk_starts
    assert g.size == 0 or int(g.max()) < 256
    gaps[:n_chunks] = g.astype(np.uint8)
    block_starts = np.arange(n_blocks, dtype=np.uint64) * np.uint64(threads_per_block * chunk_bits)
    blkoff = np.zeros(n_blocks + 1, np.uint64)
    blkoff[:n_blocks] = np.searchsorted(starts[:n], block_starts, side="left")
    blkoff[n_blocks] = n
    return n_chunks, n_blocks, gaps, blkoff


def encode(w: np.ndarray, chunk_bytes: int = DEFAULT_CHUNK_BYTES,
           threads_per_block: int = DEFAULT_THREADS_PER_BLOCK,
           max_len: int = DEFAULT_MAX_LEN) -> np.ndarray:
    """Compress BF16 bit patterns into a DFloat11 blob (uint8 array)."""
    if chunk_bytes % 4 or chunk_bytes < 8 or threads_per_block % 32 or not 32 <= threads_per_block <= 1024:
        raise ValueError("bad chunk/block parameters")
    if not 1 <= max_len <= FORMAT_MAX_LEN:
        raise ValueError("bad length limit")
    w = np.ascontiguousarray(w, dtype=np.uint16).reshape(-1)
    n = w.size
    e, s = split(w)
    counts = histogram(e)
    present = H.present_symbols(counts)
    lengths = H.limited_lengths(counts, max_len)
    header = dict(magic=B.MAGIC, version=B.VERSION, codec=B.CODEC_DFLOAT11, n=n,
                  header_bytes=B.HEADER_BYTES, chunk_bytes=chunk_bytes,
                  threads_per_block=threads_per_block)
    len_arr = np.array(lengths, np.uint8)
    sm = np.zeros(B.align(n, 16), np.uint8)
    sm[:n] = s
    if len(present) <= 1:
        header.update(flags=B.FLAG_SINGLE_EXPONENT if n else 0,
                      const_exp=present[0] if present else 0)
        sections = [("lengths", len_arr), ("lut", np.zeros(0, np.uint16)),
                    ("gaps", np.zeros(0, np.uint8)), ("blkoff", np.zeros(0, np.uint64)),
                    ("stream", np.zeros(0, np.uint32)), ("sm", sm)]
        return B.assemble(header, sections)

    codes = H.canonical_codes(lengths)
    tables = H.build_lut(lengths)
    total_bits = int(sum(int(counts[i]) * lengths[i] for i in range(256)))
    n_words = -(-total_bits // 32)
    stream_bytes = B.align(4 * n_words + 16, 16)
    words = np.zeros(stream_bytes // 4, np.uint32)
    code_arr = np.array(codes, np.uint32)
    written = lib().orc_df11_emit(ptr(e, ctypes.c_uint8), n, ptr(len_arr, ctypes.c_uint8),
                                  ptr(code_arr, ctypes.c_uint32), ptr(words, ctypes.c_uint32))
    assert written == total_bits
    chunk_bits = 8 * chunk_bytes
    n_chunks, n_blocks, gaps, blkoff = chunk_index(len_arr[e], total_bits, chunk_bits,
                                                   threads_per_block)
    header.update(flags=0, max_len=max(lengths), n_tables=len(tables), n_chunks=n_chunks,
                  n_blocks=n_blocks, total_bits=total_bits,
                  max_block_count=int(np.diff(blkoff).max()), const_exp=0,
                  stream_bytes=stream_bytes)
    sections = [("lengths", len_arr), ("lut", np.array(tables, np.uint16).reshape(-1)),
                ("gaps", gaps), ("blkoff", blkoff), ("stream", words), ("sm", sm)]
    return B.assemble(header, sections)


def _parts(blob: np.ndarray, h: dict):
    n = h["n"]
    sm = B.section(blob, h["off_sm"], B.align(n, 16))[:n]
    lengths = [int(x) for x in B.section(blob, h["off_lengths"], 256)]
    return sm, lengths


def decode_exponents(blob: np.ndarray, h: dict | None = None, want_lengths: bool = False):
    """Sequential bit-serial decode of all n exponents (and their code lengths)."""
    blob = np.asarray(blob, np.uint8)
    h = h or B.unpack_header(blob)
    n = h["n"]
    if h["flags"] & B.FLAG_SINGLE_EXPONENT or n == 0:
        e = np.full(n, h["const_exp"], np.uint8)
        return (e, np.zeros(n, np.uint8)) if want_lengths else e
    _, lengths = _parts(blob, h)
    if max(lengths) > FORMAT_MAX_LEN:
        raise ValueError("code longer than the format allows")
    if H.kraft_numerator(lengths) > 1 << 32:
        raise ValueError("code lengths violate the Kraft inequality")
    first, cnt, base, sorted_syms = H.decode_tables(lengths)
    words = B.section(blob, h["off_stream"], h["stream_bytes"], np.uint32)
    if h["total_bits"] > 32 * words.size:
        raise ValueError("stream section shorter than total_bits")
    e = np.empty(n, np.uint8)
    lens = np.empty(n, np.uint8) if want_lengths else None
    f = np.array(first, np.uint32)
    c = np.array(cnt, np.uint32)
    b = np.array(base, np.uint32)
    ss = np.array(sorted_syms + [0], np.uint8)
    end = ctypes.c_uint64(0)
    rc = lib().orc_df11_decode_syms(ptr(words, ctypes.c_uint32), h["total_bits"], 0, n,
                                    ptr(f, ctypes.c_uint32), ptr(c, ctypes.c_uint32),
                                    ptr(b, ctypes.c_uint32), ptr(ss, ctypes.c_uint8), 32,
                                    ptr(e, ctypes.c_uint8), ptr(lens, ctypes.c_uint8),
                                    ctypes.byref(end))
    if rc != 0:
        raise ValueError(f"corrupt stream (code {rc} at bit {end.value})")
    if end.value != h["total_bits"]:
        raise ValueError("stream longer than its n codes")
    return (e, lens) if want_lengths else e


def decode(blob: np.ndarray) -> np.ndarray:
    """Decompress a DFloat11 blob back to the BF16 bit patterns (uint16)."""
    blob = np.asarray(blob, np.uint8)
    h = B.unpack_header(blob)
    if h["codec"] != B.CODEC_DFLOAT11:
        raise ValueError("not a DFloat11 blob")
    e = decode_exponents(blob, h)
    sm, _ = _parts(blob, h)
    return merge(e, np.ascontiguousarray(sm))


def check_index(blob: np.ndarray) -> list[str]:
    """Re-derive gaps, blkoff, max_block_count and the lookup tables of a blob
    from its sequential decode and code lengths; list every disagreement."""
    blob = np.asarray(blob, np.uint8)
    h = B.unpack_header(blob)
    problems = []
    if h["flags"] & B.FLAG_SINGLE_EXPONENT or h["n"] == 0:
        if h["n_blocks"] or h["total_bits"]:
            problems.append("single-exponent blob with a stream")
        return problems
    e, lens = decode_exponents(blob, h, want_lengths=True)
    T, C = h["threads_per_block"], h["chunk_bytes"]
    n_chunks, n_blocks, gaps, blkoff = chunk_index(lens, h["total_bits"], 8 * C, T)
    if (n_chunks, n_blocks) != (h["n_chunks"], h["n_blocks"]):
        problems.append("chunk/block counts")
        return problems
    stored_gaps = B.section(blob, h["off_gaps"], n_blocks * T)
    stored_blk = B.section(blob, h["off_blkoff"], 8 * (n_blocks + 1), np.uint64)
    if not np.array_equal(stored_gaps, gaps):
        problems.append("gaps")
    if not np.array_equal(stored_blk, blkoff):
        problems.append("blkoff")
    if int(np.diff(blkoff).max()) != h["max_block_count"]:
        problems.append("max_block_count")
    _, lengths = _parts(blob, h)
    if max(lengths) != h["max_len"]:
        problems.append("max_len")
    lut = B.section(blob, h["off_lut"], 512 * h["n_tables"], np.uint16).reshape(-1, 256).tolist()
    codes = H.canonical_codes(lengths)
    for sym in range(256):
        l = lengths[sym]
        if l and H.lut_lookup(lut, codes[sym] << (32 - l)) != (sym, l):
            problems.append(f"lut entry for exponent {sym}")
            break
    return problems


def bits_per_weight(blob: np.ndarray) -> float:
    h = B.unpack_header(blob)
    return 8.0 * h["total_bytes"] / max(1, h["n"])
