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
  weight it decodes (``blkoff``). Optionally (``chunk_counts``) it also
  carries, per chunk, the number of codes that start in it (``counts``):
  the result of the first phase, worked out once by the encoder, so that a
  decoder can go straight to the scan and the writing phase.

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


def chunk_output_offsets(code_lengths_per_weight: np.ndarray, total_bits: int, chunk_bits: int,
                         threads_per_block: int) -> np.ndarray:
    """Per chunk, where its codes' outputs start inside its block: the number
    of codes of the block that start before the chunk's first code (its gap).
    This is the result of the two-phase decoder's first phase plus the block
    scan (DFloat11 page, "Jak to działa w praktyce?": each thread first learns
    how much it decodes, then writes at its place), i.e. what a blob would
    store to let the decoder skip that phase. Chunks past the stream end get
    their block's code count."""
    n = code_lengths_per_weight.size
    starts = np.zeros(n + 1, np.uint64)
    np.cumsum(code_lengths_per_weight, dtype=np.uint64, out=starts[1:])
    assert int(starts[-1]) == total_bits
    n_chunks, n_blocks, _, blkoff = chunk_index(code_lengths_per_weight, total_bits, chunk_bits, threads_per_block)
    first = np.full(n_blocks * threads_per_block, n, np.uint64)   # index of each chunk's first code
    chunk_starts = np.arange(n_chunks, dtype=np.uint64) * np.uint64(chunk_bits)
    first[:n_chunks] = np.searchsorted(starts[:n], chunk_starts, side="left")
    block_of = np.arange(n_blocks * threads_per_block) // threads_per_block
    first = np.minimum(first, blkoff[block_of + 1])
    return (first - blkoff[block_of]).astype(np.uint32)


def chunk_output_offsets_of_blob(blob: np.ndarray) -> np.ndarray:
    """chunk_output_offsets for a DFloat11 blob, from its sequential decode."""
    blob = np.asarray(blob, np.uint8)
    h = B.unpack_header(blob)
    if h["codec"] != B.CODEC_DFLOAT11:
        raise ValueError("not a DFloat11 blob")
    if h["total_bits"] == 0:
        return np.zeros(0, np.uint32)
    _, lens = decode_exponents(blob, h, want_lengths=True)
    return chunk_output_offsets(np.asarray(lens, np.uint64), h["total_bits"], 8 * h["chunk_bytes"],
                                h["threads_per_block"])


def chunk_code_counts(code_lengths_per_weight: np.ndarray, total_bits: int, chunk_bits: int,
                      threads_per_block: int) -> np.ndarray:
    """Per chunk, the number of codes that start in it: #{i < n : c*chunk_bits
    <= starts[i] < (c+1)*chunk_bits}, starts[i] being the exclusive prefix sum
    of the code lengths. This is what each thread finds in the first phase of
    the two-phase decoder (DFloat11 page, "Jak to działa w praktyce?": threads
    first learn how much they will decode). The array covers n_blocks *
    threads_per_block chunks; chunks at or past the stream end count 0."""
    n = code_lengths_per_weight.size
    starts = np.zeros(n + 1, np.uint64)
    np.cumsum(code_lengths_per_weight, dtype=np.uint64, out=starts[1:])
    assert int(starts[-1]) == total_bits
    n_chunks = -(-total_bits // chunk_bits)
    n_blocks = -(-n_chunks // threads_per_block)
    chunk_of = (starts[:n] // np.uint64(chunk_bits)).astype(np.int64)
    return np.bincount(chunk_of, minlength=n_blocks * threads_per_block).astype(np.uint64)


def counts_fit_in_bytes(lengths, chunk_bits: int) -> bool:
    """Whether every per-chunk code count fits in a byte for this code: codes
    are at least min_len bits long, so at most ceil(chunk_bits / min_len) of
    them start in one chunk."""
    present = [l for l in lengths if l > 0]
    return bool(present) and -(-chunk_bits // min(present)) <= 255


def encode(w: np.ndarray, chunk_bytes: int = DEFAULT_CHUNK_BYTES,
           threads_per_block: int = DEFAULT_THREADS_PER_BLOCK,
           max_len: int = DEFAULT_MAX_LEN, _elem: int = B.ELEM_BF16, _lo=None,
           chunk_counts: bool = True) -> np.ndarray:
    """Compress BF16 bit patterns into a DFloat11 blob (uint8 array).

    With ``chunk_counts`` the blob also stores each chunk's code count (a
    byte per chunk, flag FLAG_CHUNK_COUNTS) whenever every count fits in a
    byte (``counts_fit_in_bytes``); otherwise it is left out.
    (``_elem`` / ``_lo`` are used by ``encode_elements`` for FP32 and FP16:
    the element type recorded in the header and the low-mantissa section.)"""
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
                  threads_per_block=threads_per_block, elem=_elem)
    lo_sections = [] if _lo is None else [("lo", _lo)]
    if _lo is not None:
        header["lo_bytes"] = _lo.nbytes
    len_arr = np.array(lengths, np.uint8)
    sm = np.zeros(B.align(n, 16), np.uint8)
    sm[:n] = s
    if len(present) <= 1:
        header.update(flags=B.FLAG_SINGLE_EXPONENT if n else 0,
                      const_exp=present[0] if present else 0)
        sections = [("lengths", len_arr), ("lut", np.zeros(0, np.uint16)),
                    ("gaps", np.zeros(0, np.uint8)), ("blkoff", np.zeros(0, np.uint64)),
                    ("stream", np.zeros(0, np.uint32)), ("sm", sm)] + lo_sections
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
    with_counts = chunk_counts and counts_fit_in_bytes(lengths, chunk_bits)
    header.update(flags=B.FLAG_CHUNK_COUNTS if with_counts else 0, max_len=max(lengths),
                  n_tables=len(tables), n_chunks=n_chunks,
                  n_blocks=n_blocks, total_bits=total_bits,
                  max_block_count=int(np.diff(blkoff).max()), const_exp=0,
                  stream_bytes=stream_bytes)
    count_sections = []
    if with_counts:
        counts = chunk_code_counts(len_arr[e], total_bits, chunk_bits, threads_per_block)
        assert int(counts.max()) <= 255
        count_sections = [("counts", counts.astype(np.uint8))]
    sections = [("lengths", len_arr), ("lut", np.array(tables, np.uint16).reshape(-1)),
                ("gaps", gaps)] + count_sections + [("blkoff", blkoff), ("stream", words),
                                                    ("sm", sm)] + lo_sections
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
    """Decompress a DFloat11 blob back to the BF16 bit patterns (uint16).
    For FP32 / FP16 blobs this is the intermediate 16-bit pattern; use
    ``decode_elements`` for the elements themselves."""
    blob = np.asarray(blob, np.uint8)
    h = B.unpack_header(blob)
    if h["codec"] != B.CODEC_DFLOAT11:
        raise ValueError("not a DFloat11 blob")
    e = decode_exponents(blob, h)
    sm, _ = _parts(blob, h)
    return merge(e, np.ascontiguousarray(sm))


def decode_blocks(blob: np.ndarray, b0: int, b1: int) -> np.ndarray:
    """Weights blkoff[b0] .. blkoff[b1] of a DFloat11 blob, decoded bit-serially
    from the first code of block b0 (its chunk's gap) without touching the
    blocks before it: the independence the stored block offsets and gaps give
    (DFloat11 page, "Jak to działa w praktyce?"), used to spread the decode of
    one tensor over several processes."""
    blob = np.asarray(blob, np.uint8)
    h = B.unpack_header(blob)
    if h["codec"] != B.CODEC_DFLOAT11:
        raise ValueError("not a DFloat11 blob")
    if h["flags"] & B.FLAG_SINGLE_EXPONENT or h["n"] == 0:
        if (b0, b1) != (0, 0):
            raise ValueError("a blob without a stream has no blocks")
        return decode(blob)
    if not 0 <= b0 <= b1 <= h["n_blocks"]:
        raise ValueError("block range outside the blob")
    T, cb = h["threads_per_block"], 8 * h["chunk_bytes"]
    blkoff = B.section(blob, h["off_blkoff"], 8 * (h["n_blocks"] + 1), np.uint64)
    gaps = B.section(blob, h["off_gaps"], h["n_blocks"] * T)
    i0, i1 = int(blkoff[b0]), int(blkoff[b1])
    if i1 == i0:
        return np.zeros(0, np.uint16)
    _, lengths = _parts(blob, h)
    first, cnt, base, sorted_syms = H.decode_tables(lengths)
    words = B.section(blob, h["off_stream"], h["stream_bytes"], np.uint32)
    e = np.empty(i1 - i0, np.uint8)
    f = np.array(first, np.uint32)
    c = np.array(cnt, np.uint32)
    bb = np.array(base, np.uint32)
    ss = np.array(sorted_syms + [0], np.uint8)
    end = ctypes.c_uint64(0)
    start = b0 * T * cb + int(gaps[b0 * T])
    rc = lib().orc_df11_decode_syms(ptr(words, ctypes.c_uint32), h["total_bits"], start, i1 - i0,
                                    ptr(f, ctypes.c_uint32), ptr(c, ctypes.c_uint32),
                                    ptr(bb, ctypes.c_uint32), ptr(ss, ctypes.c_uint8), 32,
                                    ptr(e, ctypes.c_uint8), None, ctypes.byref(end))
    if rc != 0:
        raise ValueError(f"corrupt stream (code {rc} at bit {end.value})")
    sm, _ = _parts(blob, h)
    return merge(e, np.ascontiguousarray(sm[i0:i1]))


# ---------------------------------------------------------------- FP32 and FP16
#
# The DFloat11 idea carried to the other float formats: entropy-code the
# exponent, keep sign and mantissa as they are. Each element is mapped to a
# 16-bit pattern laid out like BF16 (sign, 8-bit exponent field, 7 mantissa
# bits), which goes through the BF16 codec above, plus the mantissa bits that
# do not fit, stored raw in a "lo" section:
#  * FP32 (1 + 8 + 23 bits): the top 16 bits are exactly a BF16 pattern; the
#    low 16 mantissa bits are stored as uint16.
#  * FP16 (1 + 5 + 10 bits): the pattern is sign | exponent (0..31, in the
#    8-bit field) | top 7 mantissa bits; the low 3 mantissa bits are packed,
#    3 bits per weight, least significant bits first.

def split_elements(x: np.ndarray, elem: int):
    """(v, lo): the BF16-shaped 16-bit patterns and the raw low mantissa bits."""
    if elem == B.ELEM_BF16:
        return np.ascontiguousarray(x, np.uint16).reshape(-1), None
    if elem == B.ELEM_FP32:
        x = np.ascontiguousarray(x, np.uint32).reshape(-1)
        return (x >> 16).astype(np.uint16), (x & 0xFFFF).astype(np.uint16)
    if elem == B.ELEM_FP16:
        x = np.ascontiguousarray(x, np.uint16).reshape(-1).astype(np.uint32)
        sign, expo, mant = x >> 15, (x >> 10) & 0x1F, x & 0x3FF
        v = (sign << 15) | (expo << 7) | (mant >> 3)
        return v.astype(np.uint16), (mant & 7).astype(np.uint8)
    raise ValueError(f"unknown element type {elem}")


def merge_elements(v: np.ndarray, lo, elem: int) -> np.ndarray:
    """Inverse of split_elements."""
    v = np.asarray(v, np.uint16)
    if elem == B.ELEM_BF16:
        return v.copy()
    if elem == B.ELEM_FP32:
        return (v.astype(np.uint32) << 16) | np.asarray(lo, np.uint32)
    if elem == B.ELEM_FP16:
        v = v.astype(np.uint32)
        sign, expo, mant7 = v >> 15, (v >> 7) & 0xFF, v & 0x7F
        if expo.size and int(expo.max()) > 0x1F:
            raise ValueError("FP16 exponent field above 31")
        return ((sign << 15) | (expo << 10) | (mant7 << 3) | np.asarray(lo, np.uint32)).astype(np.uint16)
    raise ValueError(f"unknown element type {elem}")


def pack3(lo: np.ndarray) -> np.ndarray:
    """3-bit values, value i at stream bits 3i..3i+2 (bit b of the stream is
    bit b mod 8 of byte b / 8)."""
    lo = np.asarray(lo, np.uint8).reshape(-1)
    bits = ((lo[:, None] >> np.arange(3, dtype=np.uint8)) & 1).reshape(-1)
    return np.packbits(bits, bitorder="little")


def unpack3(packed: np.ndarray, n: int) -> np.ndarray:
    bits = np.unpackbits(np.asarray(packed, np.uint8), bitorder="little")[:3 * n].reshape(n, 3)
    return (bits * np.array([1, 2, 4], np.uint8)).sum(axis=1).astype(np.uint8)


def lo_section(lo, elem: int, n: int) -> np.ndarray:
    """The raw low-mantissa section: FP32 uint16[n], FP16 packed 3-bit values;
    padded with zeros to a multiple of 16 bytes, with at least 16 bytes after
    the FP16 values."""
    if elem == B.ELEM_FP32:
        out = np.zeros(B.align(2 * n, 16), np.uint8)
        out[:2 * n] = np.asarray(lo, np.uint16).view(np.uint8)
        return out
    packed = pack3(lo)
    out = np.zeros(B.align(-(-3 * n // 8) + 16, 16), np.uint8)
    out[:packed.size] = packed
    return out


def encode_elements(x: np.ndarray, elem: int, chunk_bytes: int = DEFAULT_CHUNK_BYTES,
                    threads_per_block: int = DEFAULT_THREADS_PER_BLOCK,
                    max_len: int = DEFAULT_MAX_LEN) -> np.ndarray:
    """DFloat11 blob of FP32 (uint32 patterns), FP16 or BF16 (uint16) elements."""
    v, lo = split_elements(x, elem)
    if elem == B.ELEM_BF16:
        return encode(v, chunk_bytes, threads_per_block, max_len)
    return encode(v, chunk_bytes, threads_per_block, max_len, _elem=elem,
                  _lo=lo_section(lo, elem, v.size))


def decode_elements(blob: np.ndarray) -> np.ndarray:
    """The elements of a DFloat11 blob of any element type (uint32 for FP32,
    uint16 otherwise)."""
    blob = np.asarray(blob, np.uint8)
    h = B.unpack_header(blob)
    elem, n = h["elem"], h["n"]
    v = decode(blob)
    if elem == B.ELEM_BF16:
        return v
    raw = B.section(blob, h["off_lo"], h["lo_bytes"])
    if elem == B.ELEM_FP32:
        if h["lo_bytes"] < 2 * n:
            raise ValueError("low-mantissa section too short")
        lo = raw[:2 * n].view(np.uint16)
    elif elem == B.ELEM_FP16:
        if h["lo_bytes"] < -(-3 * n // 8):
            raise ValueError("low-mantissa section too short")
        lo = unpack3(raw, n)
    else:
        raise ValueError(f"unknown element type {elem}")
    return merge_elements(v, lo, elem)


def check_index(blob: np.ndarray) -> list[str]:
    """Re-derive gaps, blkoff, max_block_count, the per-chunk code counts (if
    stored) and the lookup tables of a blob from its sequential decode and
    code lengths; list every disagreement."""
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
    if h["flags"] & B.FLAG_CHUNK_COUNTS:
        stored_counts = B.section(blob, h["off_counts"], n_blocks * T)
        if not np.array_equal(stored_counts.astype(np.uint64), chunk_code_counts(lens, h["total_bits"], 8 * C, T)):
            problems.append("counts")
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
