"""Pins of the oracle against facts that do not come from the oracle itself:
the identity (decode must return the input, bit for bit), closed forms,
textbook optimality by brute force, the pages' aggregate figures, and
hand-derived worked examples under tests/golden/."""
import itertools
import math

import numpy as np
import pytest

import synth
from conftest import load_golden
from oracle import blob as B
from oracle import codebook, df11
from oracle import huffman as H


def hexes(xs):
    return np.array([int(x, 16) for x in xs], np.uint16)


# ---------------------------------------------------------------- identity

def roundtrip_both(w, **kw):
    b = df11.encode(w, **kw)
    assert np.array_equal(df11.decode(b), w)
    assert df11.check_index(b) == []
    c = codebook.encode(w)
    assert np.array_equal(codebook.decode(c), w)
    return b, c


def test_roundtrip_small_square():
    w = synth.as_u16(synth.small_square(0))
    roundtrip_both(w)


def test_all_65536_patterns():
    w = synth.as_u16(synth.all_patterns())
    b, c = roundtrip_both(w)
    h = B.unpack_header(b)
    assert h["n_tables"] == 1 and h["max_len"] == 8   # 256 equiprobable exponents -> 8-bit codes
    hc = B.unpack_header(c)
    assert (hc["U"], hc["k"]) == (65536, 16)


def test_tiny_tensors_bruteforce():
    # every tensor of length <= 4 over {+0, -0, a NaN with payload}
    alphabet = [0x0000, 0x8000, 0x7FC1]
    for length in range(0, 5):
        for combo in itertools.product(alphabet, repeat=length):
            w = np.array(combo, np.uint16)
            roundtrip_both(w, chunk_bytes=8, threads_per_block=32)


@pytest.mark.parametrize("n", list(range(0, 34)) + [255, 256, 257, 1000])
def test_random_lengths(n):
    w = synth.as_u16(synth.uniform_patterns(n, seed=100 + n))
    roundtrip_both(w, chunk_bytes=8, threads_per_block=32)


@pytest.mark.parametrize("chunk_bytes,tpb", [(8, 32), (12, 64), (36, 256), (64, 128), (252, 1024)])
def test_chunk_parameters(chunk_bytes, tpb):
    w = synth.as_u16(synth.normal_bf16((200_003,), seed=7, sigma=0.02, outlier_frac=1e-3))
    roundtrip_both(w, chunk_bytes=chunk_bytes, threads_per_block=tpb)


def test_single_exponent_and_empty():
    for w in (np.zeros(1000, np.uint16), np.full(37, 0x3F80, np.uint16), np.zeros(0, np.uint16)):
        b, c = roundtrip_both(w)
        h = B.unpack_header(b)
        assert h["total_bits"] == 0 and h["n_blocks"] == 0
    # same exponent, different signs and mantissas: still one exponent symbol
    w = (np.arange(5000, dtype=np.uint16) & 0x807F) | 0x3F00
    b, _ = roundtrip_both(w)
    h = B.unpack_header(b)
    assert h["flags"] & B.FLAG_SINGLE_EXPONENT and h["const_exp"] == 126


def test_uniform_exponents_maximal_spread():
    # exponents uniform over all 256 values: every code is 8 bits, stream = 8 bits/weight
    w = synth.as_u16(synth.uniform_patterns(1 << 18, seed=3))
    b, _ = roundtrip_both(w)
    counts, lengths, _ = df11.code_for(w)
    assert H.entropy_bits(counts) > 7.99
    assert all(l in (7, 8, 9) for l in lengths)
    # 8 raw bits + 8 code bits, plus a gap byte and a count byte per 36-byte
    # chunk of 36 codes (2 x 8/36 = 0.44 bits), the block offsets and the
    # 256-byte section alignment (about 0.05 bits at this size)
    assert 15.9 < df11.bits_per_weight(b) < 16.6


@pytest.mark.parametrize("L", range(1, 9))
def test_flat_histograms_give_fixed_length_affine_codes(L):
    """2^L consecutive exponents in equal numbers: Huffman merges them in
    pairs level by level, so every code word has length L, and canonical codes
    of one length follow symbol order, so exponent e0 + v gets word v; the
    stream is then L-bit fields, weight i's at bits [iL, iL + L). This is what
    the decoder's fixed-length path relies on."""
    w = synth.as_u16(synth.equal_exponents(2048 * (1 << L) + 5, L, seed=L))
    counts, lengths, _ = df11.code_for(w)
    present = [e for e in range(256) if lengths[e]]
    e0 = present[0]
    assert present == list(range(e0, e0 + (1 << L)))
    assert {lengths[e] for e in present} == {L}
    codes = H.canonical_codes(lengths)
    assert [codes[e] for e in present] == list(range(1 << L))
    b = df11.encode(w)
    h = B.unpack_header(b)
    assert h["total_bits"] == L * w.size
    words = B.section(b, h["off_stream"], h["stream_bytes"], np.uint32)
    bits = "".join(format(int(x), "032b") for x in words[: (L * w.size + 31) // 32])
    e = (w >> 7) & 0xFF
    for i in list(range(0, w.size, 97)) + [w.size - 1]:
        assert int(bits[i * L:(i + 1) * L], 2) == int(e[i]) - e0, i


def test_unequal_histogram_is_not_fixed_length():
    # counts 4000 : 1000 : 1000 : 1000 over four exponents: lengths (1, 2, 3, 3)
    # cost 12,000 bits against 14,000 for four 2-bit codes, so the code has
    # several lengths and the fixed-length path must not apply
    w = np.repeat(np.array([120, 121, 122, 123], np.uint16) << 7, [4000, 1000, 1000, 1000])
    counts, lengths, _ = df11.code_for(w)
    assert sorted(l for l in lengths if l) == [1, 2, 3, 3]


# ------------------------------------------------------- code properties

def code_strings(lengths, codes):
    return sorted(format(codes[s], f"0{l}b") for s, l in enumerate(lengths) if l)


def assert_complete_prefix_free(lengths, max_len=32):
    codes = H.canonical_codes(lengths)
    strs = code_strings(lengths, codes)
    for a, b in zip(strs, strs[1:]):
        assert not b.startswith(a), (a, b)
    if len(strs) >= 2:
        assert H.kraft_numerator(lengths, 32) == 1 << 32
    assert max(lengths) <= max_len


@pytest.mark.parametrize("seed", range(6))
def test_kraft_and_prefix_free(seed):
    rng = np.random.default_rng(seed)
    m = int(rng.integers(2, 257))
    counts = np.zeros(256, np.uint64)
    syms = rng.choice(256, m, replace=False)
    counts[syms] = rng.geometric(0.05, m) ** 3      # very skewed counts
    assert_complete_prefix_free(H.huffman_lengths(counts), max_len=64)
    assert_complete_prefix_free(H.limited_lengths(counts, 12), max_len=12)


def test_fibonacci_counts_need_the_length_limit():
    # Fibonacci counts make the Huffman tree a path: depth = alphabet size - 1
    fib = [1, 1]
    while len(fib) < 40:
        fib.append(fib[-1] + fib[-2])
    counts = np.zeros(256, np.uint64)
    counts[:40] = fib
    assert max(H.huffman_lengths(counts)) == 39
    lim = H.limited_lengths(counts, 32)
    assert max(lim) == 32
    assert_complete_prefix_free(lim)
    w = np.repeat((np.arange(40, dtype=np.uint16) << 7), np.array(fib[:40]) % 50 + 1)
    roundtrip_both(w)


def brute_force_min_cost(c, max_len):
    best = None
    for ls in itertools.product(range(1, max_len + 1), repeat=len(c)):
        if sum(2.0 ** -l for l in ls) <= 1.0:
            cost = sum(ci * li for ci, li in zip(c, ls))
            best = cost if best is None else min(best, cost)
    return best


@pytest.mark.parametrize("seed", range(12))
def test_huffman_optimal_bruteforce(seed):
    rng = np.random.default_rng(1000 + seed)
    m = int(rng.integers(2, 8))
    c = [int(x) for x in rng.integers(1, 60, m)]
    counts = np.zeros(256, np.uint64)
    syms = sorted(rng.choice(256, m, replace=False).tolist())
    counts[syms] = c
    lengths = H.huffman_lengths(counts)
    cost = sum(int(counts[s]) * lengths[s] for s in syms)
    assert cost == brute_force_min_cost(c, m - 1)


@pytest.mark.parametrize("seed", range(12))
def test_length_limited_optimal_bruteforce(seed):
    rng = np.random.default_rng(2000 + seed)
    m = int(rng.integers(3, 7))
    L = int(rng.integers(math.ceil(math.log2(m)), m))
    c = [int(x) for x in rng.geometric(0.3, m) ** 2]
    counts = np.zeros(256, np.uint64)
    syms = sorted(rng.choice(256, m, replace=False).tolist())
    counts[syms] = c
    lengths = H.package_merge(counts, L)
    assert max(lengths) <= L
    assert sum(2.0 ** -lengths[s] for s in syms) <= 1.0
    cost = sum(int(counts[s]) * lengths[s] for s in syms)
    assert cost == brute_force_min_cost(c, L)


def test_package_merge_matches_huffman_when_unconstrained():
    rng = np.random.default_rng(5)
    for _ in range(5):
        counts = np.zeros(256, np.uint64)
        counts[rng.choice(256, 30, replace=False)] = rng.integers(1, 1000, 30)
        hl = H.huffman_lengths(counts)
        pm = H.package_merge(counts, 32)
        cost = lambda ls: sum(int(counts[s]) * ls[s] for s in range(256))
        assert cost(hl) == cost(pm)


def test_entropy_bounds_and_page_figures():
    # DFloat11 page, "Przełom: DFloat11": the exponent carries about 2.6 bits
    # and the compressed model is about 70 % of BF16, about 11 bits/weight.
    w = synth.as_u16(synth.small_square(0))
    counts, lengths, _ = df11.code_for(w)
    ent = H.entropy_bits(counts)
    avg = H.average_length(counts, lengths)
    assert ent <= avg < ent + 1.0                       # Shannon / Huffman bound
    assert 2.1 < ent < 3.1                              # "about 2.6 bits"
    b = df11.encode(w)
    bpw = df11.bits_per_weight(b)
    assert 10.0 < bpw < 11.5                            # "about 11 bits"
    assert 0.62 < bpw / 16 < 0.72                       # "about 70 %"


def test_stream_length_is_sum_of_count_times_length():
    w = synth.as_u16(synth.normal_bf16((100_000,), seed=11, sigma=0.03, outlier_frac=1e-3))
    counts, lengths, _ = df11.code_for(w)
    b = df11.encode(w)
    h = B.unpack_header(b)
    assert h["total_bits"] == sum(int(counts[s]) * lengths[s] for s in range(256))


def test_sign_and_mantissa_untouched():
    # DFloat11 page, "Przełom: DFloat11": sign and mantissa are stored as they are
    w = synth.as_u16(synth.uniform_patterns(4096, seed=9))
    b = df11.encode(w)
    h = B.unpack_header(b)
    sm = B.section(b, h["off_sm"], h["n"])
    assert np.array_equal(sm >> 7, (w >> 15).astype(np.uint8))
    assert np.array_equal(sm & 0x7F, (w & 0x7F).astype(np.uint8))


# ------------------------------------------------ chunked (two-phase) view

def decode_chunk(words, total_bits, start, end, lengths):
    """Codes starting in [start, end): what one GPU thread decodes."""
    import ctypes
    from oracle._native import lib, ptr
    first, cnt, base, sorted_syms = H.decode_tables(lengths)
    f, c, bb = (np.array(x, np.uint32) for x in (first, cnt, base))
    ss = np.array(sorted_syms + [0], np.uint8)
    out = []
    pos = start
    sym = np.zeros(1, np.uint8)
    endbit = ctypes.c_uint64()
    while pos < end:
        rc = lib().orc_df11_decode_syms(ptr(words, ctypes.c_uint32), total_bits, pos, 1,
                                        ptr(f, ctypes.c_uint32), ptr(c, ctypes.c_uint32),
                                        ptr(bb, ctypes.c_uint32), ptr(ss, ctypes.c_uint8), 32,
                                        ptr(sym, ctypes.c_uint8), None, ctypes.byref(endbit))
        assert rc == 0
        out.append(int(sym[0]))
        pos = endbit.value
    return out


@pytest.mark.parametrize("chunk_bytes,tpb", [(8, 32), (36, 64)])
def test_chunks_decode_independently(chunk_bytes, tpb):
    """Decoding every chunk from its own gap, as the two-phase GPU decoder
    does, yields the whole exponent sequence, and each block's count matches
    blkoff (DFloat11 page, "Jak to działa w praktyce?": threads count first,
    then write at the right place)."""
    w = synth.as_u16(synth.normal_bf16((40_000,), seed=21, sigma=0.02, outlier_frac=2e-3))
    b = df11.encode(w, chunk_bytes=chunk_bytes, threads_per_block=tpb)
    h = B.unpack_header(b)
    e_ref, _ = df11.split(w)
    lengths = [int(x) for x in B.section(b, h["off_lengths"], 256)]
    words = B.section(b, h["off_stream"], h["stream_bytes"], np.uint32)
    gaps = B.section(b, h["off_gaps"], h["n_blocks"] * tpb)
    blkoff = B.section(b, h["off_blkoff"], 8 * (h["n_blocks"] + 1), np.uint64)
    cb = 8 * chunk_bytes
    got = []
    for blk in range(h["n_blocks"]):
        in_block = 0
        for t in range(tpb):
            c = blk * tpb + t
            start = c * cb + int(gaps[c])
            end = min((c + 1) * cb, h["total_bits"])
            syms = decode_chunk(words, h["total_bits"], start, end, lengths)
            in_block += len(syms)
            got.extend(syms)
        assert in_block == int(blkoff[blk + 1] - blkoff[blk])
    assert np.array_equal(np.array(got, np.uint8), e_ref)


@pytest.mark.parametrize("chunk_bytes,tpb", [(8, 32), (36, 32), (36, 64)])
def test_chunk_output_offsets_match_independent_chunk_decodes(chunk_bytes, tpb):
    """The per-chunk output offsets a blob could store (the first phase plus
    the block scan, done once by the encoder) equal the running code count of
    each block when every chunk is decoded on its own from its gap."""
    w = synth.as_u16(synth.normal_bf16((30_000,), seed=23, sigma=0.02, outlier_frac=3e-3))
    b = df11.encode(w, chunk_bytes=chunk_bytes, threads_per_block=tpb)
    h = B.unpack_header(b)
    offs = df11.chunk_output_offsets_of_blob(b)
    assert offs.size == h["n_blocks"] * tpb
    lengths = [int(x) for x in B.section(b, h["off_lengths"], 256)]
    words = B.section(b, h["off_stream"], h["stream_bytes"], np.uint32)
    gaps = B.section(b, h["off_gaps"], h["n_blocks"] * tpb)
    blkoff = B.section(b, h["off_blkoff"], 8 * (h["n_blocks"] + 1), np.uint64)
    cb = 8 * chunk_bytes
    for blk in range(h["n_blocks"]):
        running = 0
        for t in range(tpb):
            c = blk * tpb + t
            assert offs[c] == running, (blk, t)
            if c * cb < h["total_bits"]:
                running += len(decode_chunk(words, h["total_bits"], c * cb + int(gaps[c]),
                                            min((c + 1) * cb, h["total_bits"]), lengths))
        assert running == int(blkoff[blk + 1] - blkoff[blk])


def test_chunk_output_offsets_single_code_length():
    # all 16 exponents equally frequent: every code is 4 bits, so chunk c's
    # first code is code ceil(c * cb / 4) and its offset is that minus the
    # block's first code (closed form, no decode)
    e = np.repeat(np.arange(120, 136, dtype=np.uint16), 1000)
    w = ((np.random.default_rng(3).permutation(e) << 7) | 0x0011).astype(np.uint16)
    for chunk_bytes, tpb in ((8, 32), (36, 64)):
        b = df11.encode(w, chunk_bytes=chunk_bytes, threads_per_block=tpb)
        h = B.unpack_header(b)
        assert h["max_len"] == 4 and h["total_bits"] == 4 * w.size
        offs = df11.chunk_output_offsets_of_blob(b)
        cb = 8 * chunk_bytes
        for c in range(offs.size):
            blk = c // tpb
            first = min(-(-c * cb // 4), w.size)
            blk_first = min(-(-blk * tpb * cb // 4), w.size)
            assert offs[c] == first - blk_first


@pytest.mark.parametrize("chunk_bytes,tpb", [(8, 32), (36, 32), (36, 64)])
def test_chunk_counts_match_independent_chunk_decodes(chunk_bytes, tpb):
    """The per-chunk code counts a blob stores equal the number of codes each
    chunk yields when it is decoded on its own, from its gap up to the next
    chunk's first code (what each thread of the two-phase decoder counts in
    the first phase), and each block's counts add up to its stored offsets."""
    w = synth.as_u16(synth.normal_bf16((30_000,), seed=29, sigma=0.02, outlier_frac=3e-3))
    b = df11.encode(w, chunk_bytes=chunk_bytes, threads_per_block=tpb)
    h = B.unpack_header(b)
    assert h["flags"] & B.FLAG_CHUNK_COUNTS
    counts = B.section(b, h["off_counts"], h["n_blocks"] * tpb)
    lengths = [int(x) for x in B.section(b, h["off_lengths"], 256)]
    words = B.section(b, h["off_stream"], h["stream_bytes"], np.uint32)
    gaps = B.section(b, h["off_gaps"], h["n_blocks"] * tpb)
    blkoff = B.section(b, h["off_blkoff"], 8 * (h["n_blocks"] + 1), np.uint64)
    cb, tb = 8 * chunk_bytes, h["total_bits"]
    for c in range(h["n_blocks"] * tpb):
        got = len(decode_chunk(words, tb, c * cb + int(gaps[c]), min((c + 1) * cb, tb), lengths)) \
            if c * cb < tb else 0
        assert counts[c] == got, c
    sums = counts.astype(np.int64).reshape(-1, tpb).sum(axis=1)
    assert np.array_equal(sums, np.diff(blkoff.astype(np.int64)))


def test_chunk_counts_single_code_length():
    # all 16 exponents equally frequent: every code is 4 bits, so the codes
    # that start in chunk c are the multiples of 4 in [c cb, min((c+1) cb, TB)):
    # ceil(min((c+1) cb, TB) / 4) - ceil(c cb / 4) of them (closed form, no decode)
    e = np.repeat(np.arange(120, 136, dtype=np.uint16), 1000)
    w = ((np.random.default_rng(5).permutation(e) << 7) | 0x0033).astype(np.uint16)
    for chunk_bytes, tpb in ((8, 32), (20, 32), (36, 64)):
        b = df11.encode(w, chunk_bytes=chunk_bytes, threads_per_block=tpb)
        h = B.unpack_header(b)
        assert h["max_len"] == 4 and h["flags"] & B.FLAG_CHUNK_COUNTS
        counts = B.section(b, h["off_counts"], h["n_blocks"] * tpb)
        cb, tb = 8 * chunk_bytes, h["total_bits"]
        for c in range(counts.size):
            lo, hi = min(c * cb, tb), min((c + 1) * cb, tb)
            assert counts[c] == -(-hi // 4) - -(-lo // 4), c


def test_chunk_counts_only_when_they_fit_a_byte():
    # exponent 126 in 3/4 of the weights gets a 1-bit code, so up to 288 codes
    # can start in a 288-bit chunk: more than a byte counts, and the counts
    # are left out; in 64-bit chunks at most 64 start, and they are stored
    rng = np.random.default_rng(6)
    e = rng.choice(np.array([126, 125, 127], np.uint16), size=20_000, p=[0.75, 0.125, 0.125])
    w = ((e << 7) | rng.integers(0, 256, e.size, dtype=np.uint16) & 0x807F).astype(np.uint16)
    lengths = df11.code_for(w)[1]
    assert min(l for l in lengths if l) == 1
    wide = df11.encode(w, chunk_bytes=36, threads_per_block=32)
    assert not B.unpack_header(wide)["flags"] & B.FLAG_CHUNK_COUNTS
    narrow = df11.encode(w, chunk_bytes=8, threads_per_block=32)
    assert B.unpack_header(narrow)["flags"] & B.FLAG_CHUNK_COUNTS
    assert df11.check_index(narrow) == [] and np.array_equal(df11.decode(narrow), w)
    off = df11.encode(w, chunk_bytes=8, threads_per_block=32, chunk_counts=False)
    assert not B.unpack_header(off)["flags"] & B.FLAG_CHUNK_COUNTS
    assert np.array_equal(df11.decode(off), w)


@pytest.mark.parametrize("chunk_bytes,tpb", [(8, 64), (36, 32), (36, 256)])
def test_block_ranges_decode_independently(chunk_bytes, tpb):
    """Any split of a blob's blocks into ranges, each decoded from its own
    first gap, concatenates to the whole tensor (what lets one tensor's decode
    be spread over processes)."""
    w = synth.as_u16(synth.normal_bf16((120_007,), seed=31, sigma=0.02, outlier_frac=2e-3))
    b = df11.encode(w, chunk_bytes=chunk_bytes, threads_per_block=tpb)
    nb = B.unpack_header(b)["n_blocks"]
    rng = np.random.default_rng(tpb)
    for _ in range(3):
        cuts = sorted({0, nb, *rng.integers(0, nb + 1, 4).tolist()})
        parts = [df11.decode_blocks(b, x, y) for x, y in zip(cuts[:-1], cuts[1:])]
        assert np.array_equal(np.concatenate(parts), w)
    assert df11.decode_blocks(b, 3, 3).size == 0
    with pytest.raises(ValueError):
        df11.decode_blocks(b, 2, nb + 1)
    single = np.full(1000, 0x3C12, np.uint16)
    assert np.array_equal(df11.decode_blocks(df11.encode(single), 0, 0), single)


# ----------------------------------------------------- worked examples

def test_golden_df11_worked_example():
    g = load_golden("df11_worked_example.json")
    w = hexes(g["tensor_hex"])
    e, s = df11.split(w)
    assert e.tolist() == g["exponents"]
    assert s.tolist() == [int(x, 16) for x in g["sm_hex"]]
    counts, lengths, codes = df11.code_for(w)
    for sym, l in g["lengths"].items():
        assert lengths[int(sym)] == l
        assert codes[int(sym)] == g["codes"][sym]
    b = df11.encode(w, chunk_bytes=8, threads_per_block=32)
    h = B.unpack_header(b)
    assert h["total_bits"] == g["total_bits"]
    words = B.section(b, h["off_stream"], h["stream_bytes"], np.uint32)
    assert words[0] == int(g["stream_word0"], 16)
    assert np.all(words[1:] == 0)
    assert np.array_equal(df11.decode(b), w)


def test_golden_df11_periodic_offsets():
    g = load_golden("df11_worked_example.json")
    p = g["periodic"]
    w = np.concatenate([hexes([p["lead_hex"]]), np.tile(hexes(g["tensor_hex"]), p["reps"])])
    b = df11.encode(w, chunk_bytes=p["chunk_bytes"], threads_per_block=p["threads_per_block"])
    h = B.unpack_header(b)
    assert (h["n"], h["total_bits"], h["n_chunks"], h["n_blocks"]) == (
        p["n"], p["total_bits"], p["n_chunks"], p["n_blocks"])
    blkoff = B.section(b, h["off_blkoff"], 8 * (h["n_blocks"] + 1), np.uint64)
    assert blkoff.tolist() == p["blkoff"]
    gaps = B.section(b, h["off_gaps"], h["n_blocks"] * p["threads_per_block"])
    assert gaps[:3].tolist() == p["gaps_first3"]
    # every gap from the period structure: code starts are lead 0, then
    # lead_bits + period*r + pattern_starts
    cb = 8 * p["chunk_bytes"]
    starts = [0] + [p["lead_bits"] + p["period_bits"] * r + o
                    for r in range(p["reps"]) for o in p["pattern_starts"]] + [p["total_bits"]]
    for c in range(p["n_chunks"]):
        nxt = min(x for x in starts if x >= c * cb)
        assert gaps[c] == nxt - c * cb
    assert np.all(gaps[p["n_chunks"]:] == 0)
    # per-chunk code counts: the first three by hand, all from the period structure
    assert h["flags"] & B.FLAG_CHUNK_COUNTS
    counts = B.section(b, h["off_counts"], h["n_blocks"] * p["threads_per_block"])
    assert counts[:3].tolist() == p["counts_first3"]
    for c in range(counts.size):
        assert counts[c] == sum(1 for x in starts[:-1] if c * cb <= x < (c + 1) * cb)


def _runs_to_table(runs):
    t = [None] * 256
    for lo, hi, v in runs:
        for i in range(lo, hi + 1):
            t[i] = v
    assert None not in t
    return t


def test_golden_lookup_tables():
    """Every entry of the hierarchical lookup tables (not only each code's
    first one) against tables derived by hand: the worked example's single
    table, and a two-level code with 9- and 10-bit codes behind a pointer."""
    g = load_golden("df11_worked_example.json")
    lengths = [0] * 256
    for sym, l in g["lengths"].items():
        lengths[int(sym)] = l
    tables = H.build_lut(lengths)
    assert len(tables) == 1
    assert tables[0] == _runs_to_table(g["lut"]["worked_example_table0"]["runs"])
    two = g["lut"]["two_level"]
    lengths = [0] * 256
    for sym, l in two["lengths"].items():
        lengths[int(sym)] = l
    tables = H.build_lut(lengths)
    assert len(tables) == len(two["tables"])
    for got, runs in zip(tables, two["tables"]):
        assert got == _runs_to_table(runs)


def test_lut_lookup_matches_prefix_search():
    """lut_lookup on every 16-bit stream prefix returns the one code that is
    a prefix of it, found by comparing the prefix with every codeword
    (brute force), for the two-level golden code and a 4-level code."""
    g = load_golden("df11_worked_example.json")["lut"]["two_level"]
    two = [0] * 256
    for sym, l in g["lengths"].items():
        two[int(sym)] = l
    fib = [0] * 256                       # Fibonacci-like lengths 1..24, 25: a path 4 tables deep
    for i in range(24):
        fib[100 + i] = i + 1
    fib[124] = 24
    for lengths in (two, fib):
        codes = H.canonical_codes(lengths)
        tables = H.build_lut(lengths)
        rng = np.random.default_rng(7)
        xs = (np.arange(1 << 16, dtype=np.uint64) << np.uint64(16)) | rng.integers(0, 1 << 16, 1 << 16).astype(np.uint64)
        want_sym = np.full(xs.size, -1, np.int64)
        want_len = np.zeros(xs.size, np.int64)
        for sym in range(256):
            if lengths[sym]:
                hit = (xs >> np.uint64(32 - lengths[sym])) == np.uint64(codes[sym])
                assert not np.any(hit & (want_sym >= 0))     # prefix-free: one code per prefix
                want_sym[hit], want_len[hit] = sym, lengths[sym]
        assert np.all(want_sym >= 0)                          # complete: every prefix starts a code
        for x, ws, wl in zip(xs.tolist(), want_sym.tolist(), want_len.tolist()):
            assert H.lut_lookup(tables, x) == (ws, wl), hex(x)


def test_golden_clrs_huffman():
    g = load_golden("df11_worked_example.json")["clrs"]
    counts = np.zeros(256, np.uint64)
    for sym, c in g["counts"].items():
        counts[int(sym)] = c
    lengths = H.huffman_lengths(counts)
    codes = H.canonical_codes(lengths)
    for sym, l in g["lengths"].items():
        assert lengths[int(sym)] == l
        assert codes[int(sym)] == g["canonical_codes"][sym]
    assert sum(int(counts[s]) * lengths[s] for s in range(256)) == g["cost"]


def test_golden_codebook_worked_example():
    g = load_golden("codebook_worked_example.json")
    w = hexes(g["tensor_hex"])
    b = codebook.encode(w)
    h = B.unpack_header(b)
    assert (h["U"], h["k"]) == (g["U"], g["k"])
    table = B.section(b, h["off_table"], 2 * h["U"], np.uint16)
    assert table.tolist() == [int(x, 16) for x in g["table_hex"]]
    words = B.section(b, h["off_packed"], h["packed_bytes"], np.uint32)
    assert words[0] == int(g["packed_word0"], 16)
    assert np.array_equal(codebook.decode(b), w)
    for U, k in g["index_bits_cases"]:
        assert codebook.index_bits(U) == k


# ------------------------------------------------------------- codebook

@pytest.mark.parametrize("U", [1, 2, 3, 5, 255, 256, 257, 4096, 8192])
def test_codebook_table_and_width(U):
    w = synth.as_u16(synth.codebook_stress(U, 50_000, seed=U))
    b = codebook.encode(w)
    h = B.unpack_header(b)
    distinct = set(int(x) for x in w.tolist())          # brute-force count
    assert h["U"] == len(distinct)
    assert h["k"] == (0 if h["U"] <= 1 else (h["U"] - 1).bit_length())
    table = B.section(b, h["off_table"], 2 * h["U"], np.uint16).tolist()
    assert table == sorted(distinct)
    assert np.array_equal(codebook.decode(b), w)
    # every weight read on its own gives the same value
    idx = np.random.default_rng(U).integers(0, w.size, 200)
    for i in idx.tolist():
        assert codebook.decode_range(b, i, 1)[0] == w[i]


def test_codebook_bits_per_weight_closed_form():
    w = synth.as_u16(synth.codebook_stress(4096, 1 << 20, seed=4))
    b = codebook.encode(w)
    h = B.unpack_header(b)
    payload_bits = h["k"] * h["n"] + 16 * h["U"]
    assert h["k"] == 12
    assert payload_bits <= 8 * h["total_bytes"] <= payload_bits + 8 * (256 * 4 + 16)


# ---------------------------------------------------------------- FP32 / FP16 elements
#
# The oracle's element split must agree with the IEEE formats themselves:
# each finite normal element's value is rebuilt, in float64, from the parts
# the split produces (sign, exponent field, mantissa bits) and compared with
# numpy's own reading of the same bits; the exponent field is compared with
# frexp. A wrong bit position or field width fails here.

def _rebuild(sign, expo, mant, bias, mant_bits):
    return np.where(sign == 1, -1.0, 1.0) * (1.0 + mant / float(1 << mant_bits)) * np.exp2(expo.astype(np.float64) - bias)


def test_fp16_split_matches_ieee_half():
    x = np.arange(65536, dtype=np.uint16)
    v, lo = df11.split_elements(x, B.ELEM_FP16)
    sign = (v >> 15).astype(np.int64)
    expo = ((v >> 7) & 0xFF).astype(np.int64)
    mant = (((v & 0x7F).astype(np.int64)) << 3) | lo.astype(np.int64)
    val = x.view(np.float16).astype(np.float64)
    normal = (expo >= 1) & (expo <= 30)
    assert expo.max() <= 31
    assert np.array_equal(_rebuild(sign, expo, mant, 15, 10)[normal], val[normal])
    _, e2 = np.frexp(val[normal])
    assert np.array_equal(expo[normal], e2 - 1 + 15)
    assert np.array_equal(df11.merge_elements(v, lo, B.ELEM_FP16), x)


def test_fp32_split_matches_ieee_single():
    rng = np.random.default_rng(5)
    x = rng.integers(0, 2 ** 32, 200_000, dtype=np.uint64).astype(np.uint32)
    v, lo = df11.split_elements(x, B.ELEM_FP32)
    sign = (v >> 15).astype(np.int64)
    expo = ((v >> 7) & 0xFF).astype(np.int64)
    mant = (((v & 0x7F).astype(np.int64)) << 16) | lo.astype(np.int64)
    val = x.view(np.float32).astype(np.float64)
    normal = (expo >= 1) & (expo <= 254)
    assert np.array_equal(_rebuild(sign, expo, mant, 127, 23)[normal], val[normal])
    _, e2 = np.frexp(val[normal])
    assert np.array_equal(expo[normal], e2 - 1 + 127)
    assert np.array_equal(df11.merge_elements(v, lo, B.ELEM_FP32), x)


def test_pack3_is_little_endian_bit_concatenation():
    rng = np.random.default_rng(6)
    for n in (1, 2, 3, 7, 8, 9, 100):
        vals = rng.integers(0, 8, n)
        as_int = sum(int(v) << (3 * i) for i, v in enumerate(vals))
        expect = np.frombuffer(as_int.to_bytes(-(-3 * n // 8), "little"), np.uint8)
        got = df11.pack3(vals)
        assert np.array_equal(got, expect), n
        assert np.array_equal(df11.unpack3(got, n), vals.astype(np.uint8))


def test_element_blobs_round_trip_and_entropy():
    x16 = synth.as_u16(synth.normal_fp16((200_000,), seed=3, sigma=0.02))
    b = df11.encode_elements(x16, B.ELEM_FP16, threads_per_block=32)
    assert np.array_equal(df11.decode_elements(b), x16)
    h = B.unpack_header(b)
    assert h["elem"] == B.ELEM_FP16 and h["lo_bytes"] >= -(-3 * x16.size // 8)
    # only the 32 FP16 exponent values can have codes; Huffman within 1 bit of the entropy
    v, _ = df11.split_elements(x16, B.ELEM_FP16)
    e, _ = df11.split(v)
    counts = df11.histogram(e)
    assert counts[32:].sum() == 0
    lengths = [int(x) for x in B.section(b, h["off_lengths"], 256)]
    p = counts[counts > 0] / counts.sum()
    entropy = float(-(p * np.log2(p)).sum())
    avg = float(sum(int(counts[i]) * lengths[i] for i in range(256)) / counts.sum())
    assert entropy <= avg < entropy + 1
    x32 = (np.random.default_rng(8).standard_normal(100_001).astype(np.float32) * 0.02).view(np.uint32)
    b = df11.encode_elements(x32, B.ELEM_FP32, threads_per_block=32)
    assert np.array_equal(df11.decode_elements(b), x32)
    assert 8.0 * b.size / x32.size < 28.0    # exponent coded, 24 raw bits kept
