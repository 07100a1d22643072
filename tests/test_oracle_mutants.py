"""Strength of the oracle's pins: each test plants one plausible mistake in
the oracle (on the CPU, by monkeypatching a single function) and checks that
a pin from test_oracle_pins.py then fails."""
import numpy as np
import pytest

import test_oracle_pins as pins
from oracle import codebook, df11
from oracle import huffman as H


def fails(fn, *args):
    with pytest.raises((AssertionError, ValueError)):
        fn(*args)


def test_canonical_without_shift_is_caught(monkeypatch):
    def bad(lengths):
        order = sorted((l, s) for s, l in enumerate(lengths) if l > 0)
        codes = [0] * 256
        for i, (_, s) in enumerate(order):
            codes[s] = i                       # forgets the shift on a length change
        return codes
    monkeypatch.setattr(H, "canonical_codes", bad)
    fails(pins.test_golden_df11_worked_example)
    fails(pins.test_golden_clrs_huffman)


def test_depth_off_by_one_is_caught(monkeypatch):
    good = H.huffman_lengths
    monkeypatch.setattr(H, "huffman_lengths", lambda c: [l + 1 if l else 0 for l in good(c)])
    fails(pins.test_huffman_optimal_bruteforce, 0)
    fails(pins.test_golden_clrs_huffman)


def test_package_merge_selection_off_by_one_is_caught(monkeypatch):
    good = H.package_merge

    def bad(counts, max_len):
        out = good(counts, max_len)
        syms = [s for s in range(256) if out[s]]
        out[syms[0]] += 1                        # as if one extra item were selected
        return out
    monkeypatch.setattr(H, "package_merge", bad)
    fails(pins.test_length_limited_optimal_bruteforce, 0)


def test_floor_log2_width_is_caught(monkeypatch):
    monkeypatch.setattr(codebook, "index_bits", lambda U: max(0, U.bit_length() - 1))
    fails(pins.test_golden_codebook_worked_example)
    fails(pins.test_codebook_table_and_width, 3)


def test_gap_off_by_one_is_caught(monkeypatch):
    good = df11.chunk_index

    def bad(lens, total_bits, chunk_bits, tpb):
        n_chunks, n_blocks, gaps, blkoff = good(lens, total_bits, chunk_bits, tpb)
        gaps = gaps.copy()
        gaps[1:n_chunks] += 1
        return n_chunks, n_blocks, gaps, blkoff
    monkeypatch.setattr(df11, "chunk_index", bad)
    fails(pins.test_chunks_decode_independently, 8, 32)
    fails(pins.test_golden_df11_periodic_offsets)


def test_chunk_counts_by_code_end_is_caught(monkeypatch):
    def bad(lens, total_bits, chunk_bits, tpb):
        # counts the codes that end in each chunk instead of those that start there
        ends = np.cumsum(np.asarray(lens, np.uint64), dtype=np.uint64)
        n_blocks = -(-(-(-total_bits // chunk_bits)) // tpb)
        chunk_of = ((ends - np.uint64(1)) // np.uint64(chunk_bits)).astype(np.int64)
        return np.bincount(chunk_of, minlength=n_blocks * tpb).astype(np.uint64)
    monkeypatch.setattr(df11, "chunk_code_counts", bad)
    fails(pins.test_golden_df11_periodic_offsets)
    fails(pins.test_chunk_counts_match_independent_chunk_decodes, 8, 32)


def _build_lut_with(fill_delta=0, pointer_delta=0):
    """build_lut with one planted mistake: the fill count of every leaf off
    by fill_delta, or the table index stored in new pointers off by
    pointer_delta."""
    def build(lengths):
        codes = H.canonical_codes(lengths)
        order = sorted((l, s) for s, l in enumerate(lengths) if l > 0)
        tables = [[H.LUT_INVALID] * 256]
        for l, s in order:
            c, t, depth = codes[s], 0, 0
            while l > 8 * (depth + 1):
                prefix = (c >> (l - 8 * (depth + 1))) & 0xFF
                entry = tables[t][prefix]
                if entry == H.LUT_INVALID:
                    tables.append([H.LUT_INVALID] * 256)
                    entry = 0x8000 | (len(tables) - 1 + pointer_delta)
                    tables[t][prefix] = entry
                t = min(entry & 0x7FFF, len(tables) - 1)
                depth += 1
            rest = l - 8 * depth
            low = c & ((1 << rest) - 1)
            for fill in range(max(1, (1 << (8 - rest)) + fill_delta)):
                tables[t][((low << (8 - rest)) | fill) & 0xFF] = (l << 8) | s
        return tables
    return build


def test_lut_fill_count_off_by_one_is_caught(monkeypatch):
    monkeypatch.setattr(H, "build_lut", _build_lut_with(fill_delta=-1))
    fails(pins.test_golden_lookup_tables)
    fails(pins.test_lut_lookup_matches_prefix_search)


def test_lut_pointer_off_by_one_is_caught(monkeypatch):
    monkeypatch.setattr(H, "build_lut", _build_lut_with(pointer_delta=1))
    fails(pins.test_golden_lookup_tables)
    fails(pins.test_lut_lookup_matches_prefix_search)


def test_dropped_sign_is_caught(monkeypatch):
    good = df11.merge
    monkeypatch.setattr(df11, "merge", lambda e, s: good(e, s & np.uint8(0x7F)))
    fails(pins.test_roundtrip_small_square)
    fails(pins.test_all_65536_patterns)


def test_swapped_exponent_and_mantissa_split_is_caught(monkeypatch):
    good = df11.split

    def bad(w):
        e, s = good(w)
        return e, (s & 0x80) | ((s & 0x7F)[::-1].copy())   # mantissas in the wrong order
    monkeypatch.setattr(df11, "split", bad)
    fails(pins.test_sign_and_mantissa_untouched)


def test_lsb_msb_confusion_in_codebook_is_caught(monkeypatch):
    good = codebook.encode

    def bad(w):
        b = good(w)
        from oracle import blob as B
        h = B.unpack_header(b)
        off = h["off_packed"]
        n = h["packed_bytes"]
        # reverse the bit order inside each byte (MSB-first packing)
        bits = np.unpackbits(b[off:off + n]).reshape(-1, 8)[:, ::-1]
        b[off:off + n] = np.packbits(bits.reshape(-1))
        return b
    monkeypatch.setattr(codebook, "encode", bad)
    fails(pins.test_golden_codebook_worked_example)


def test_fp16_exponent_off_by_one_bit_is_caught(monkeypatch):
    good = df11.split_elements

    def bad(x, elem):
        if elem != 2:
            return good(x, elem)
        x = np.ascontiguousarray(x, np.uint16).astype(np.uint32)
        sign, expo, mant = x >> 15, (x >> 11) & 0x1F, x & 0x3FF      # exponent read one bit too high
        return ((sign << 15) | (expo << 7) | (mant >> 3)).astype(np.uint16), (mant & 7).astype(np.uint8)
    monkeypatch.setattr(df11, "split_elements", bad)
    fails(pins.test_fp16_split_matches_ieee_half)


def test_fp32_halves_swapped_is_caught(monkeypatch):
    good = df11.split_elements

    def bad(x, elem):
        if elem != 1:
            return good(x, elem)
        x = np.ascontiguousarray(x, np.uint32)
        return (x & 0xFFFF).astype(np.uint16), (x >> 16).astype(np.uint16)   # high and low halves swapped
    monkeypatch.setattr(df11, "split_elements", bad)
    fails(pins.test_fp32_split_matches_ieee_single)


def test_pack3_msb_first_is_caught(monkeypatch):
    def bad(lo):
        lo = np.asarray(lo, np.uint8).reshape(-1)
        bits = ((lo[:, None] >> np.arange(3, dtype=np.uint8)[::-1]) & 1).reshape(-1)   # bits reversed
        return np.packbits(bits, bitorder="little")
    monkeypatch.setattr(df11, "pack3", bad)
    fails(pins.test_pack3_is_little_endian_bit_concatenation)


# ---- linear-layer oracle (oracle/linear.py) ----------------------------------

import test_oracle_linear as lpins
from oracle import linear as OL


def _bad_linear(transform):
    def bad(w_bits, x_bits):
        w = OL.bf16_values(w_bits)
        x = OL.bf16_values(x_bits)
        w, x = transform(w, x)
        return x @ w.T, np.abs(x) @ np.abs(w).T
    return bad


def test_linear_transposed_operand_is_caught(monkeypatch):
    monkeypatch.setattr(OL, "linear", lambda w_bits, x_bits: (
        OL.bf16_values(x_bits) @ OL.bf16_values(w_bits), np.abs(OL.bf16_values(x_bits)) @ np.abs(OL.bf16_values(w_bits))))
    fails(lpins.test_golden_square_example_catches_a_transpose)


def test_linear_shifted_column_is_caught(monkeypatch):
    monkeypatch.setattr(OL, "linear", _bad_linear(lambda w, x: (w, np.roll(x, 1, axis=1))))
    fails(lpins.test_one_hot_selects_a_column, 6)
    fails(lpins.test_golden_rectangular_example)


def test_linear_dropped_last_column_is_caught(monkeypatch):
    monkeypatch.setattr(OL, "linear", _bad_linear(lambda w, x: (w[:, :-1], x[:, :-1])))
    fails(lpins.test_ones_closed_form)
    fails(lpins.test_exact_rational_sums, 0)


def test_bf16_exponent_bias_off_by_one_is_caught(monkeypatch):
    good = OL.bf16_values
    monkeypatch.setattr(OL, "bf16_values", lambda b: good(b) * 0.5)
    fails(lpins.test_bf16_field_values)
    fails(lpins.test_bf16_values_match_float32_upper_half_on_every_pattern)


def test_bf16_sign_dropped_is_caught(monkeypatch):
    good = OL.bf16_values
    monkeypatch.setattr(OL, "bf16_values", lambda b: np.abs(good(b)))
    fails(lpins.test_bf16_field_values)
    fails(lpins.test_golden_rectangular_example)


def test_chunk_offsets_off_by_one_is_caught(monkeypatch):
    good = df11.chunk_output_offsets

    def bad(*a):
        o = good(*a).copy()
        o[1:] += 1
        return o
    monkeypatch.setattr(df11, "chunk_output_offsets", bad)
    fails(pins.test_chunk_output_offsets_match_independent_chunk_decodes, 8, 32)
    fails(pins.test_chunk_output_offsets_single_code_length)


def _tile_order_by(order):
    """A tile order with the tiles or their contents walked the wrong way."""
    def f(w_bits, tile_rows=128, tile_cols=64):
        w = np.asarray(w_bits)
        rows, cols = w.shape
        pieces = []
        grid = [(i, j) for i in range(rows // tile_rows) for j in range(cols // tile_cols)]
        if order == "tiles_by_column":
            grid = [(i, j) for j in range(cols // tile_cols) for i in range(rows // tile_rows)]
        for i, j in grid:
            tile = w[i * tile_rows:(i + 1) * tile_rows, j * tile_cols:(j + 1) * tile_cols]
            pieces.append(tile.T.reshape(-1) if order == "tile_column_major" else tile.reshape(-1))
        return np.concatenate(pieces)
    return f


@pytest.mark.parametrize("order", ["tiles_by_column", "tile_column_major"])
def test_tile_order_walked_the_wrong_way_is_caught(monkeypatch, order):
    monkeypatch.setattr(OL, "tile_order", _tile_order_by(order))
    fails(lpins.test_golden_tile_order)
