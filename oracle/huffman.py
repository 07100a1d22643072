"""Oracle: Huffman code construction for the 8-bit BF16 exponent.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Follows "Koniec z kompromisami! DFloat11 ratuje dokładność modeli AI ..."
(gadzety360.pl), section "Przełom: DFloat11 – bezstratna kompresja z
wydajnością GPU": the exponent is entropy coded with a Huffman code, so that
frequent exponent values get short codes and rare ones long codes. The page
states no tie-break, no length bound and no code ordering; the readings used
here are:

* Huffman tree by the textbook greedy merge, smallest (count, id) first,
  leaves having id = symbol and internal nodes id = 256 + creation order.
* If the tree is deeper than ``max_len`` the lengths are replaced by the
  optimal length-limited ones from the package-merge algorithm
  (Larmore & Hirschberg, 1990).
* Canonical code assignment in (length, symbol) order, as in DEFLATE
  (RFC 1951, section 3.2.2).
* Hierarchical decode tables of 256 entries, each indexed by the next 8
  stream bits (section "Jak to działa w praktyce? Magia na poziomie GPU":
  several small linked lookup tables instead of one large one).
"""
from __future__ import annotations

import heapq
import math

import numpy as np

ALPHABET = 256


def present_symbols(counts) -> list[int]:
    return [s for s in range(ALPHABET) if int(counts[s]) > 0]


def huffman_lengths(counts) -> list[int]:
    """Code length of each of the 256 exponent values (0 = value absent).

    A single present value gets length 0: the stream is empty and the decoder
    repeats that value (the reading for the degenerate one-symbol alphabet).
    """
    syms = present_symbols(counts)
    lengths = [0] * ALPHABET
    if len(syms) <= 1:
        return lengths
    # heap items: (count, id, node); node = symbol (int) or (left, right)
    heap = [(int(counts[s]), s, s) for s in syms]
    heapq.heapify(heap)
    next_id = ALPHABET
    while len(heap) > 1:
        c1, _, n1 = heapq.heappop(heap)
        c2, _, n2 = heapq.heappop(heap)
        heapq.heappush(heap, (c1 + c2, next_id, (n1, n2)))
        next_id += 1
    # depth of every leaf
    stack = [(heap[0][2], 0)]
    while stack:
        node, depth = stack.pop()
        if isinstance(node, tuple):
            stack.append((node[0], depth + 1))
            stack.append((node[1], depth + 1))
        else:
            lengths[node] = depth
    return lengths


def package_merge(counts, max_len: int) -> list[int]:
    """Optimal code lengths subject to length <= max_len (package-merge).

    Coin-collector formulation: every present symbol owns one coin of each
    denomination 2^-1 .. 2^-max_len, worth its count. Starting from the
    2^-max_len coins, repeatedly pair adjacent items into packages of the next
    larger denomination and merge them with that denomination's coins, in
    ascending worth. The 2(m-1) cheapest items of denomination 2^-1 form the
    optimal selection, and a symbol's code length is the number of its coins
    in it.
    """
    syms = sorted(present_symbols(counts), key=lambda s: (int(counts[s]), s))
    m = len(syms)
    lengths = [0] * ALPHABET
    if m <= 1:
        return lengths
    if m > (1 << max_len):
        raise ValueError("alphabet too large for the length limit")

    def coin(s):
        mult = np.zeros(ALPHABET, dtype=np.int64)
        mult[s] = 1
        return (int(counts[s]), mult)

    coins = [coin(s) for s in syms]          # sorted by worth
    items = list(coins)                      # denomination 2^-max_len
    for _ in range(max_len - 1):
        packages = [(items[2 * i][0] + items[2 * i + 1][0], items[2 * i][1] + items[2 * i + 1][1])
                    for i in range(len(items) // 2)]
        merged = []
        a = b = 0
        while a < len(coins) or b < len(packages):
            if b >= len(packages) or (a < len(coins) and coins[a][0] <= packages[b][0]):
                merged.append(coins[a])
                a += 1
            else:
                merged.append(packages[b])
                b += 1
        items = merged
    total = np.zeros(ALPHABET, dtype=np.int64)
    for _, mult in items[: 2 * (m - 1)]:
        total += mult
    return [int(x) for x in total]


def limited_lengths(counts, max_len: int) -> list[int]:
    """Huffman lengths, replaced by package-merge lengths if too long."""
    lengths = huffman_lengths(counts)
    if max(lengths) > max_len:
        lengths = package_merge(counts, max_len)
    return lengths


def kraft_numerator(lengths, max_len: int = 32) -> int:
    """sum over present symbols of 2^(max_len - len); equals 2^max_len for a complete code."""
    return sum(1 << (max_len - l) for l in lengths if l > 0)


def canonical_codes(lengths) -> list[int]:
    """Canonical codewords: symbols in (length, symbol) order get consecutive
    values, each shifted left when the length grows (RFC 1951, 3.2.2)."""
    order = sorted((l, s) for s, l in enumerate(lengths) if l > 0)
    codes = [0] * ALPHABET
    code = 0
    prev = None
    for l, s in order:
        if prev is not None:
            code = (code + 1) << (l - prev)
        codes[s] = code
        prev = l
    return codes


def decode_tables(lengths, max_len: int = 32):
    """first[l], cnt[l], base[l] (l = 0..max_len) and the symbols sorted by
    (length, symbol), for bit-serial canonical decoding."""
    order = sorted((l, s) for s, l in enumerate(lengths) if l > 0)
    codes = canonical_codes(lengths)
    first = [0] * (max_len + 1)
    cnt = [0] * (max_len + 1)
    base = [0] * (max_len + 1)
    sorted_syms = [s for _, s in order]
    for i, (l, s) in enumerate(order):
        if cnt[l] == 0:
            first[l] = codes[s]
            base[l] = i
        cnt[l] += 1
    return first, cnt, base, sorted_syms


LUT_INVALID = 0xFFFF


def build_lut(lengths) -> list[list[int]]:
    """Hierarchical decode tables of 256 16-bit entries.

    Table 0 is indexed by the first 8 bits of a code; a code longer than 8
    bits continues in a table indexed by its next 8 bits, and so on. Entry:
    leaf = (length << 8) | symbol, with bit 15 clear, length = the whole code
    length; pointer = 0x8000 | table index; unused = 0xFFFF.
    """
    codes = canonical_codes(lengths)
    order = sorted((l, s) for s, l in enumerate(lengths) if l > 0)
    tables = [[LUT_INVALID] * 256]
    for l, s in order:
        c = codes[s]
        t = 0
        depth = 0
        while l > 8 * (depth + 1):
            prefix = (c >> (l - 8 * (depth + 1))) & 0xFF
            entry = tables[t][prefix]
            if entry == LUT_INVALID:
                tables.append([LUT_INVALID] * 256)
                entry = 0x8000 | (len(tables) - 1)
                tables[t][prefix] = entry
            assert entry & 0x8000, "prefix of a longer code is itself a code"
            t = entry & 0x7FFF
            depth += 1
        rest = l - 8 * depth                      # 1..8 bits left in this table
        low = c & ((1 << rest) - 1)
        for fill in range(1 << (8 - rest)):
            idx = (low << (8 - rest)) | fill
            assert tables[t][idx] == LUT_INVALID, "codes overlap"
            tables[t][idx] = (l << 8) | s
    return tables


def lut_lookup(tables, bits32: int):
    """Walk the tables with the next 32 stream bits (MSB first); returns
    (symbol, length) or None for an invalid path."""
    t = 0
    for depth in range(4):
        idx = (bits32 >> (24 - 8 * depth)) & 0xFF
        entry = tables[t][idx]
        if entry == LUT_INVALID:
            return None
        if not entry & 0x8000:
            return entry & 0xFF, (entry >> 8) & 0x3F
        t = entry & 0x7FFF
        if t >= len(tables):
            return None
    return None


def entropy_bits(counts) -> float:
    """Shannon entropy (bits/symbol) of the empirical exponent distribution."""
    total = sum(int(c) for c in counts)
    h = 0.0
    for c in counts:
        c = int(c)
        if c:
            p = c / total
            h -= p * math.log2(p)
    return h


def average_length(counts, lengths) -> float:
    total = sum(int(c) for c in counts)
    return sum(int(c) * l for c, l in zip(counts, lengths)) / total
