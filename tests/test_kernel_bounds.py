"""Index arithmetic of the decode-fused codebook linear kernel, restated and
checked on the CPU over random and extreme shapes: every bulk copy starts on a
16-byte boundary inside the packed section, ends inside it, fits the warp's
window buffer, and covers every bit a lane's fields need; every lane's word
reads stay inside the buffer; the swizzled activation slots stay inside the
staged region and are a permutation within each window (no two chunks share
a slot). The constants and formulas mirror csrc/lwc_codebook.cu
(issue_window, the re-alignment in cb_linear_kernel, stage_activations).
Also the multiply-shift division by cols of the DFloat11 linear kernel
(csrc/lwc_df11.cu: division_magic, div_cols), exact over its range."""
import numpy as np
import pytest

TILE = 1024            # indices per window (32 lanes x 32)


def buf_bytes(K):
    return 128 * K + 48


def packed_bytes(n, K):
    return (-(-n * K // 8) + 16 + 15) // 16 * 16


def window(r, q, cols, n, K):
    """(a0, bytes, boff, cnt) of window q of row r, as issue_window computes them."""
    e0 = r * cols + q * TILE
    cnt = min(TILE, cols - q * TILE)
    bit0 = e0 * K
    a0 = (bit0 >> 3) & ~15
    need = (bit0 + cnt * K + 7) // 8 + 4
    end = min((need + 15) // 16 * 16, packed_bytes(n, K))
    boff = bit0 - a0 * 8
    return a0, end - a0, boff, cnt


@pytest.mark.parametrize("K", list(range(1, 17)))
def test_window_copies_and_lane_reads_stay_in_bounds(K):
    rng = np.random.default_rng(K)
    shapes = [(1, 1), (3, 7), (5, 1023), (2, 1025), (7, 4096), (3, 14336), (1, (1 << 31) - 1)]
    shapes += [(int(rng.integers(1, 50)), int(rng.integers(1, 5000))) for _ in range(40)]
    for rows, cols in shapes:
        n = rows * cols
        pb = packed_bytes(n, K)
        nwin = -(-cols // TILE)
        for r in sorted({0, rows - 1, rows // 2}):
            for q in sorted({0, nwin - 1, nwin // 2}):
                a0, nbytes, boff, cnt = window(r, q, cols, n, K)
                assert a0 % 16 == 0 and nbytes % 16 == 0 and nbytes > 0
                assert a0 + nbytes <= pb                        # inside the packed section
                assert nbytes <= buf_bytes(K)                  # fits the window buffer
                assert 0 <= boff < 128
                # lane l reads words (boff >> 5) + l K .. + K (K + 1 words)
                last_word = (boff >> 5) + 31 * K + K
                assert 4 * (last_word + 1) <= buf_bytes(K)
                # every bit of the valid fields is inside the copied bytes
                last_field_bit = boff + cnt * K - 1
                assert last_field_bit // 8 < nbytes
                # the word after a lane's last field is read only for its low bits,
                # which belong to that lane's own fields; past the copy it is never used
                for lane in (0, 15, 31):
                    valid = max(0, min(32, cnt - 32 * lane))
                    if valid:
                        hi_bit = boff + 32 * K * lane + valid * K - 1
                        assert hi_bit // 8 < nbytes


def test_swizzled_activation_slots_are_a_permutation():
    for M, cols in ((1, 14336), (2, 4096), (8, 1024), (3, 1040), (4, 8)):
        nwin = -(-cols // TILE)
        cpr = cols // 8
        slots = []
        for m in range(M):
            for c in range(cpr):
                q, l, i = c >> 7, (c & 127) >> 2, c & 3
                slots.append((m * nwin + q) * 128 + 4 * l + ((i + (l >> 1)) & 3))
        slots = np.array(slots)
        assert np.unique(slots).size == slots.size                  # no two chunks share a slot
        assert slots.max() < M * nwin * 128                         # inside the staged region
        # the reader's view: lane l, chunk i of window q comes from (i + l / 2) & 3
        for m in range(M):
            for c in range(cpr):
                q, l, i = c >> 7, (c & 127) >> 2, c & 3
                base = (m * nwin + q) * 128 + 4 * l
                assert base + ((i + (l >> 1)) & 3) == slots[m * cpr + c]


def test_swizzle_is_bank_conflict_free_per_quarter_warp():
    # a 16-byte load by 8 lanes touches 8 distinct 16-byte bank groups
    for i in range(4):
        for quarter in range(4):
            groups = {(4 * l + ((i + (l >> 1)) & 3)) % 8 for l in range(8 * quarter, 8 * quarter + 8)}
            assert len(groups) == 8


def magic_for(d):
    """division_magic in csrc/lwc_df11.cu: l = ceil(log2 d), m' = floor(2^32 (2^l - d) / d) + 1."""
    l = 0
    while (1 << l) < d:
        l += 1
    return (((1 << l) - d) << 32) // d + 1, min(l, 1), max(l - 1, 0)


def div_cols(n, d):
    """div_cols in csrc/lwc_df11.cu: t = umulhi(m', n), q = (t + ((n - t) >> sh1)) >> sh2."""
    m, sh1, sh2 = magic_for(d)
    t = (m * n) >> 32
    return (t + ((n - t) >> sh1)) >> sh2


def test_division_by_cols_is_exact_for_every_32_bit_numerator():
    # Granlund and Montgomery's unsigned division by an invariant, as the
    # DFloat11 linear kernel uses it for rows and columns: exact for all
    # n < 2^32 and 1 <= d < 2^31, and m' fits 32 bits
    rng = np.random.default_rng(0)
    divisors = list(range(1, 70)) + [127, 128, 129, 1040, 4096, 4099, 8192, 14336, 28672, (1 << 30) + 1,
                                     (1 << 31) - 1] + [int(x) for x in rng.integers(1, 1 << 31, 200)]
    for d in divisors:
        m, _, _ = magic_for(d)
        assert 0 < m < 1 << 32
        ns = [0, 1, d - 1, d, d + 1, 2 * d - 1, (1 << 32) - 1, (1 << 32) - d, (1 << 31)]
        ns += [int(x) for x in rng.integers(0, 1 << 32, 50)]
        for n in ns:
            if 0 <= n < 1 << 32:
                assert div_cols(n, d) == n // d, (n, d)


# ---------------------------------------------------------------------------
# The DFloat11 decoder for blobs with stored chunk counts (csrc/lwc_df11.cu:
# build_counted_tables, decode_counted and the head-byte step of
# df11_counted_kernel), restated lane by lane on the CPU: its shared-memory
# stores are recorded, and the test checks that in the word phase no two
# lanes write the same staging word, that no lane writes a word holding none
# of its bytes, that every read of the segment stays inside the staged
# buffer, and that after the head-byte step the staging area holds the
# block's exponents (as the oracle decodes them, each rotated right by one
# bit, the form the merge uses).

FAST_BITS = 11
SUB_TABLES = 2


def _walk(lut, w):
    """(symbol, length) of the code at the top of the 32-bit window w, by the
    blob's hierarchical tables; None for an invalid path."""
    e = lut[w >> 24]
    d = 1
    while e & 0x8000 and d < 4:
        t = e & 0x7FFF
        if t >= len(lut) // 256:
            return None
        e = lut[t * 256 + ((w >> (24 - 8 * d)) & 0xFF)]
        d += 1
    ln = (e >> 8) & 0x3F
    if e & 0x8000 or ln == 0 or ln > 32:
        return None
    return e & 0xFF, ln


def _counted_tables(lut):
    """Symbol table (low word: up to four exponents; high word: bits used |
    8 x count << 8) and second-level tables, as build_counted_tables."""
    sym = [(0, 0)] * (1 << FAST_BITS)
    first_long = 1 << FAST_BITS
    for v in range(1 << FAST_BITS):
        w, used, cnt, syms = v << (32 - FAST_BITS), 0, 0, 0
        while cnt < 4:
            r = _walk(lut, w)
            if r is None or used + r[1] > FAST_BITS:
                break
            syms |= _rot(r[0]) << (8 * cnt)
            cnt += 1
            used += r[1]
            w = (w << r[1]) & 0xFFFFFFFF
        sym[v] = (syms, used | (8 * cnt) << 8) if cnt else (0, 0)
        if not cnt:
            first_long = min(first_long, v)
    sub = [0] * (SUB_TABLES * 256)
    for i in range(SUB_TABLES * 256):
        v = first_long + (i >> 8)
        if v < (1 << FAST_BITS):
            r = _walk(lut, (v << (32 - FAST_BITS)) | ((i & 255) << (24 - FAST_BITS)))
            if r is not None and FAST_BITS < r[1] <= FAST_BITS + 8:
                sub[i] = _rot(r[0]) | 1 << 24 | r[1] << 27
    return sym, sub, first_long


def _rot(e):
    """Exponent byte rotated right by one bit, as the tables hold it."""
    return ((e >> 1) | (e << 7)) & 0xFF


def _fsl(lo, hi, sh):
    """__funnelshift_lc: the top 32 bits of (hi:lo) << min(sh, 32)."""
    sh = min(sh, 32)
    return (((hi << 32) | lo) << sh >> 32) & 0xFFFFFFFF


def _decode_lane(seg, last, tables, pos, cnt, qb, stores, lane):
    """decode_counted for one lane: records (word, value, lane) stores into
    `stores` ('slot' for the lane's private slot); returns the stop bit."""
    sym, sub, v0 = tables
    lim = (qb + cnt + 3) >> 2
    st = {"lo": 0, "sh": (qb & 3) << 3, "nxt": (qb >> 2) + 1}
    st["dst"] = "slot" if qb & 3 else st["nxt"] - 1

    def emit(c, n8, first):
        sh = st["sh"]
        w = st["lo"] | ((c << sh) & 0xFFFFFFFF)
        spill = _fsl(c, 0, sh)
        sh += n8
        if sh >= 32:
            if first or st["nxt"] - 1 < lim:
                stores.append((st["dst"], w, lane))
            st["dst"] = st["nxt"]
            st["nxt"] += 1
            st["lo"] = spill
        else:
            st["lo"] = w
        st["sh"] = sh & 31

    def word(i):
        assert 0 <= i <= last
        return seg[i]

    k8 = cnt * 8
    while k8 > 0:
        ni = min(pos >> 5, last - 2)
        hi = _fsl(word(ni + 1), word(ni), pos & 31)
        lw = _fsl(word(ni + 2), word(ni + 1), pos & 31)
        e1 = sym[hi >> (32 - FAST_BITS)]
        if e1[1] == 0:
            s = ((hi >> (32 - FAST_BITS)) - v0) & 0xFFFFFFFF
            r = sub[(s << 8) | ((hi >> (24 - FAST_BITS)) & 0xFF)] if s < SUB_TABLES else 0
            if r == 0:
                t = _walk_or_fail(hi)
                emit(_rot(t[0]), 8, True)
                pos += t[1]
                k8 -= 8
                continue
            e1 = (r & 0xFF, (r >> 27) | 8 << 8)
        l1 = e1[1] & 31
        x2 = _fsl(lw, hi, l1)
        e2 = sym[x2 >> (32 - FAST_BITS)]
        l2 = e2[1] & 31
        e3 = sym[((x2 << l2) & 0xFFFFFFFF) >> (32 - FAST_BITS)]
        n1, n2, n3 = (e[1] >> 8 for e in (e1, e2, e3))
        emit(e1[0], n1, True)
        emit(e2[0], n2, False)
        emit(e3[0], n3, False)
        pos += l1 + l2 + (e3[1] & 31)
        k8 -= n1 + n2 + n3
    if st["nxt"] - 1 < lim:
        stores.append((st["dst"], st["lo"], lane))
    return pos


_walk_or_fail = None


@pytest.mark.parametrize("case", ["normal", "outliers", "long_codes", "chunk8"])
def test_counted_decoder_model(case):
    import synth
    from decode_dfloat11_b200 import lwc
    from oracle import blob as B
    from oracle import df11 as odf

    global _walk_or_fail
    chunk = 36
    if case == "normal":
        w = synth.as_u16(synth.normal_bf16((200_003,), seed=7, sigma=0.02, outlier_frac=1e-3))
    elif case == "outliers":
        w = synth.as_u16(synth.normal_bf16((150_001,), seed=8, sigma=0.01, outlier_frac=2e-2))
    elif case == "long_codes":   # Fibonacci counts: codes of 1..23 bits, all three lookup paths
        chunk = 8                # a 1-bit code: only chunks of <= 255 bits keep their counts
        fib = [1, 1]
        while len(fib) < 24:
            fib.append(fib[-1] + fib[-2])
        w = np.repeat((np.arange(24, dtype=np.uint16) << 7) | 0x8011, np.array(fib))
        w = np.random.default_rng(0).permutation(w).astype(np.uint16)
        firsts = np.array([int(np.argmax(w == v)) for v in np.unique(w)])   # one weight of each exponent
        w = np.concatenate([w[firsts], np.delete(w, firsts)])                # moved to block 0
    else:
        chunk = 8
        w = synth.as_u16(synth.normal_bf16((40_000,), seed=9, sigma=0.02, outlier_frac=1e-3))
    d, b = lwc.lwc_encode_dfloat11(w, chunk_bytes=chunk)
    assert d.flags & 2 and d.threads_per_block == 32
    if case == "long_codes":
        assert d.max_len == 23
    h = B.unpack_header(b)
    lut = B.section(b, h["off_lut"], 512 * h["n_tables"], np.uint16).tolist()
    tables = _counted_tables(lut)

    def walk_or_fail(wv):
        r = _walk(lut, wv)
        assert r is not None
        return r
    _walk_or_fail = walk_or_fail

    exps, _ = odf.split(w)
    words = B.section(b, h["off_stream"], h["stream_bytes"], np.uint32)
    gaps = B.section(b, h["off_gaps"], h["n_blocks"] * 32)
    counts = B.section(b, h["off_counts"], h["n_blocks"] * 32)
    blkoff = B.section(b, h["off_blkoff"], 8 * (h["n_blocks"] + 1), np.uint64)
    cw = chunk // 4
    cbits = 32 * cw
    seg_words = (32 * cw + 2 + 3) // 4 * 4
    stage_bytes = (int(np.diff(blkoff).max()) + 16 + 15) // 16 * 16
    blocks = range(h["n_blocks"]) if h["n_blocks"] <= 12 else \
        sorted({0, 1, h["n_blocks"] // 2, h["n_blocks"] - 2, h["n_blocks"] - 1})
    for blk in blocks:
        o0, o1 = int(blkoff[blk]), int(blkoff[blk + 1])
        seg0 = blk * 32 * cw
        seg = [int(x) for x in words[seg0:seg0 + seg_words]]
        seg += [0xDEADBEEF] * (seg_words - len(seg))    # stale buffer contents past the stream
        cnt = [int(c) for c in counts[blk * 32:(blk + 1) * 32]]
        first = np.concatenate([[0], np.cumsum(cnt)[:-1]]).astype(int).tolist()
        assert sum(cnt) == o1 - o0
        stores, slots = [], {}
        rem_block = h["total_bits"] - blk * 32 * cbits
        for lane in range(32):
            qb = (o0 & 15) + first[lane]
            start = lane * cbits + int(gaps[blk * 32 + lane])
            nxt_gap = int(gaps[blk * 32 + lane + 1]) if lane < 31 else \
                (int(gaps[(blk + 1) * 32]) if blk + 1 < h["n_blocks"] else 0)
            nxt = (lane + 1) * cbits + nxt_gap if (lane < 31 or blk + 1 < h["n_blocks"]) else rem_block
            end = min(nxt, rem_block)
            if cnt[lane]:
                mine = []
                got = _decode_lane(seg, seg_words - 1, tables, start, cnt[lane], qb, mine, lane)
                assert 0 <= got - end <= 40, (blk, lane, got, end)
                lo_w, hi_w = qb >> 2, (qb + cnt[lane] - 1) >> 2
                for wd, val, _ in mine:
                    if wd == "slot":
                        slots[lane] = val
                    else:
                        assert lo_w <= wd <= hi_w and (wd > lo_w or qb & 3 == 0), (blk, lane, wd)
                        assert 4 * wd + 4 <= stage_bytes
                stores += mine
        # word phase: each staging word written by one lane only
        owner = {}
        stage = bytearray(b"\xAA" * stage_bytes)
        for wd, val, lane in stores:
            if wd == "slot":
                continue
            assert owner.setdefault(wd, lane) == lane, (blk, wd)
            stage[4 * wd:4 * wd + 4] = int(val).to_bytes(4, "little")
        # head-byte step
        for lane in range(32):
            qb = (o0 & 15) + first[lane]
            if qb & 3 and cnt[lane]:
                hw, j0 = slots[lane], qb & 3
                for j in range(j0, min(4, j0 + cnt[lane])):
                    stage[(qb & ~3) + j] = (hw >> (8 * j)) & 0xFF
        got = np.frombuffer(bytes(stage[(o0 & 15):(o0 & 15) + (o1 - o0)]), np.uint8)
        assert np.array_equal(got, np.array([_rot(int(x)) for x in exps[o0:o1]], np.uint8)), blk


# ---- decode into tensor-core tiles (csrc/lwc_gemm.cu, df11_gemm_kernel) ------------
#
# Restates, on the CPU, how the decoder warps place the weights of a
# tile-order DFloat11 blob into the 128 x 64 swizzled stage tiles: each unit
# (128 rows, all columns) takes the blocks from the last one starting at or
# before its first weight to the last one starting before its end; a block
# writes its part of the unit as 8-weight pieces (one 16-byte chunk each)
# plus up to 7 single weights at either end, and adds to each tile it touches
# the number of weights it wrote there. Checked: every tile gets each of its
# 8192 slots exactly once, with the right weight, and its count reaches 8192
# exactly; a block touches at most two tiles.

def _sw128(r, c):
    return r * 128 + ((((c >> 3) ^ r) & 7) << 4) + ((c & 7) << 1)


def _last_le(blkoff, n_blocks, v):
    a, b = 0, n_blocks
    while b - a > 1:
        mid = a + (b - a) // 2
        if blkoff[mid] <= v:
            a = mid
        else:
            b = mid
    return a


def _gemm_placement(blkoff, n_blocks, tiled, rows, cols, cta_units):
    """cta_units: (128-row unit, first k-tile, k-tiles) in the CTA's order; a
    unit whose K range is split in two parts appears once per part."""
    kt = cols // 64
    slots = {}      # tile sequence number -> {byte offset: weight}
    counts = {}
    t0 = 0
    for u, kt0, kts in cta_units:
        lo = (u * kt + kt0) * 8192
        hi = lo + kts * 8192
        first, last = _last_le(blkoff, n_blocks, lo), _last_le(blkoff, n_blocks, hi - 1)
        for b in range(first, last + 1):
            o0, o1 = int(blkoff[b]), int(blkoff[b + 1])
            assert o0 <= o1 and o0 < hi and o1 > lo
            p_lo, p_hi = max(o0, lo), min(o1, hi)
            qa, qz = t0 + (p_lo - lo) // 8192, t0 + (p_hi - 1 - lo) // 8192
            assert qz - qa <= 1

            def put(i):
                t = i - lo
                q, idx = t0 + t // 8192, t % 8192
                off = _sw128(idx >> 6, idx & 63)
                assert off not in slots.setdefault(q, {})
                slots[q][off] = int(tiled[i])

            g_lo, g_hi = (p_lo + 7) & ~7, p_hi & ~7
            for pos in range(g_lo, g_hi, 8):
                t = pos - lo
                q, idx = t0 + t // 8192, t % 8192
                base = _sw128(idx >> 6, idx & 63)
                assert base % 16 == 0
                for j in range(8):   # one 16-byte chunk: weights pos .. pos + 7 in order
                    assert base + 2 * j not in slots.setdefault(q, {})
                    slots[q][base + 2 * j] = int(tiled[pos + j])
            for lane in range(16):
                i = p_lo + lane if lane < 8 else max(g_hi, g_lo) + (lane - 8)
                if (lane < 8 and i < min(g_lo, p_hi)) or (lane >= 8 and i < p_hi):
                    put(i)
            for q in range(qa, qz + 1):
                tlo = lo + (q - t0) * 8192
                counts[q] = counts.get(q, 0) + min(p_hi, tlo + 8192) - max(p_lo, tlo)
        t0 += kts
    return slots, counts


@pytest.mark.parametrize("rows,cols,chunk,order", [(384, 320, 36, "plain"), (256, 64, 8, "plain"),
                                                   (512, 192, 36, "shuffled"), (128, 1024, 12, "plain"),
                                                   (384, 320, 20, "split"), (256, 1024, 36, "split")])
def test_gemm_tile_placement_model(rows, cols, chunk, order):
    import synth
    from decode_dfloat11_b200 import lwc
    from oracle import blob as B
    from oracle import linear as OL

    w = synth.as_u16(synth.normal_bf16((rows, cols), seed=rows + cols, sigma=0.02, outlier_frac=0.01)).reshape(rows, cols)
    tiled = OL.tile_order(w)
    d, b = lwc.lwc_encode_dfloat11(tiled, chunk_bytes=chunk)
    assert d.flags & 2
    h = B.unpack_header(b)
    blkoff = B.section(b, h["off_blkoff"], 8 * (h["n_blocks"] + 1), np.uint64)
    kt = cols // 64
    units = [(u, 0, kt) for u in range(rows // 128)]
    if order == "shuffled":
        units = units[::-1]
    if order == "split":   # each unit's K range in two parts (k-tiles kt // 2 and the rest), second parts first
        half = kt // 2
        units = [(u, half, kt - half) for u in range(rows // 128)] + [(u, 0, half) for u in range(rows // 128)]
    slots, counts = _gemm_placement(blkoff, h["n_blocks"], tiled, rows, cols, units)
    n_tiles = sum(kts for _, _, kts in units)
    assert sorted(counts) == list(range(n_tiles))
    assert all(c == 8192 for c in counts.values())
    q = 0
    for u, kt0, kts in units:
        for j in range(kt0, kt0 + kts):
            assert len(slots[q]) == 8192
            for r in (0, 1, 7, 8, 63, 127):
                for c in (0, 5, 8, 31, 63):
                    assert slots[q][_sw128(r, c)] == w[u * 128 + r, j * 64 + c]
            q += 1


# ---- fixed-length codes (fixed_code_length, csrc/lwc_df11_dev.cuh; decode_fixed_range, csrc/lwc_df11.cu) ----
#
# When every code word has one length L <= 8 (flat exponent histograms: the
# uniform-exponent stress tensor is L = 8), code i is stream bits [iL, iL + L),
# and a CTA decodes the weights of its blocks straight from their indices:
# 32-weight pieces from L stream words each, the ends one by one. Restated
# here: the test that picks this path (all symbol-table entries equal), and
# the range decode, checked for in-range reads, every weight written once,
# and the exponents it produces.

def _unrot(e):
    return ((e << 1) | (e >> 7)) & 0xFF


def _fixed_code_length(sym):
    """(L, affine) as fixed_code_length decides; (0, False) for other codes."""
    y0 = sym[0][1]
    if y0 == 0 or any(e[1] != y0 for e in sym):
        return 0, False
    c, used = y0 >> 11, y0 & 31
    if c == 0 or used % c or used // c > 8:
        return 0, False
    L = used // c
    tab = [sym[v << (FAST_BITS - L)][0] & 0xFF for v in range(1 << L)]
    e0 = _unrot(tab[0])
    return L, e0 + (1 << L) - 1 <= 255 and all(_unrot(tab[v]) == e0 + v for v in range(1 << L))


def _fixed_range(words, n, L, tab, ob, oe, nt, affine=False):
    """decode_fixed_range for one CTA of nt threads: {weight: rotated exponent}
    (the affine form computes base + field and merges unrotated; returned
    rotated here, to compare alike)."""
    base = _unrot(tab[0])
    nwords = len(words)
    out = {}

    def put(i, e):
        assert ob <= i < oe and 0 <= i < n and i not in out, i
        out[i] = e

    p_lo, p_hi = (ob + 31) & ~31, oe & ~31
    for t in range(nt):
        for g in range(p_lo + 32 * t, p_hi, 32 * nt):
            w0 = g // 32 * L
            assert w0 + L <= nwords               # the piece's words exist: no read is clamped
            w = [int(words[w0 + j]) for j in range(L)] + [0]
            if affine and L == 8:   # whole bytes, byte-swapped, plus base in every byte
                for q in range(8):
                    x = int.from_bytes(w[q].to_bytes(4, "big"), "little") + base * 0x01010101
                    assert x < 1 << 32
                    for j in range(4):
                        put(g + 4 * q + j, _rot((x >> (8 * j)) & 0xFF))
                continue
            for c in range(32):
                p = c * L
                k, o = p >> 5, p & 31
                f = (((w[k] << 32 | w[k + 1]) << o) >> (64 - L)) & ((1 << L) - 1)
                assert f < len(tab)
                if affine:
                    assert base + f <= 255
                    put(g + c, _rot(base + f))
                else:
                    put(g + c, tab[f])
        for u in range(t, 62, nt):
            i = ob + u if u < 31 else max(p_hi, p_lo) + (u - 31)
            if i < min(p_lo, oe) if u < 31 else i < oe:
                p = i * L
                k = p >> 5
                wa = int(words[k]) if k < nwords else 0
                wb = int(words[k + 1]) if k + 1 < nwords else 0
                put(i, tab[_fsl(wb, wa, p & 31) >> (32 - L)])
    return out


def _blob_tables(b):
    from oracle import blob as B
    h = B.unpack_header(b)
    lut = B.section(b, h["off_lut"], 512 * h["n_tables"], np.uint16).tolist()
    return h, _counted_tables(lut)


@pytest.mark.parametrize("step", [1, 2])   # consecutive exponents (an affine code) or every other one
@pytest.mark.parametrize("L", range(1, 9))
@pytest.mark.parametrize("chunk", [8, 12, 36])
def test_fixed_length_range_model(L, chunk, step):
    import synth
    from decode_dfloat11_b200 import lwc
    from oracle import blob as B
    from oracle import df11 as odf

    if step * ((1 << L) - 1) > 255:
        pytest.skip("2^L exponents with gaps do not fit in 8 bits")
    w = synth.as_u16(synth.equal_exponents(20_001 + 37 * L, L, seed=L, step=step))
    d, b = lwc.lwc_encode_dfloat11(w, chunk_bytes=chunk)
    h, (sym, sub, first_long) = _blob_tables(b)
    lengths = B.section(b, h["off_lengths"], 256)
    assert set(lengths[lengths > 0].tolist()) == {L}
    assert first_long == 1 << FAST_BITS          # no code longer than the fast table's 11 bits
    assert _fixed_code_length(sym) == (L, step == 1)   # canonical codes of consecutive exponents
    assert h["total_bits"] == L * w.size          # the kernel's precondition holds for a valid blob
    tab = [sym[v << (FAST_BITS - L)][0] & 0xFF for v in range(1 << L)]
    exps, _ = odf.split(w)
    words = B.section(b, h["off_stream"], h["stream_bytes"], np.uint32)
    blkoff = B.section(b, h["off_blkoff"], 8 * (h["n_blocks"] + 1), np.uint64).astype(int)
    nb = h["n_blocks"]
    # CTA ranges as the launch splits the work list: G CTAs over nb blocks
    for G in (1, 3, 296):
        done = {}
        for cta in range(G):
            b0, b1 = nb * cta // G, nb * (cta + 1) // G
            if b0 >= b1:
                continue
            got = _fixed_range(words, w.size, L, tab, int(blkoff[b0]), int(blkoff[b1]), 32 if G == 3 else 576,
                               affine=_fixed_code_length(sym)[1])
            assert not (set(got) & set(done))
            done.update(got)
        assert sorted(done) == list(range(w.size))
        assert [done[i] for i in range(w.size)] == [_rot(int(x)) for x in exps]


@pytest.mark.parametrize("case", ["normal", "three_values", "nine_values", "two_lengths", "long_codes"])
def test_fixed_length_test_rejects_variable_codes(case):
    """Codes with more than one word length never take the fixed-length path,
    however flat their histogram."""
    import synth
    from decode_dfloat11_b200 import lwc

    rng = np.random.default_rng(5)
    if case == "normal":
        w = synth.as_u16(synth.normal_bf16((100_000,), seed=5, sigma=0.02))
    elif case == "long_codes":
        fib = [1, 1]
        while len(fib) < 24:
            fib.append(fib[-1] + fib[-2])
        w = np.repeat((np.arange(24, dtype=np.uint16) << 7) | 0x8011, np.array(fib))
    else:
        m = {"three_values": 3, "nine_values": 9, "two_lengths": 16}[case]
        reps = np.full(m, 1000)
        if case == "two_lengths":
            reps[:4] = 3000            # four exponents three times as frequent: lengths 3 and 5
        w = np.repeat((np.arange(120, 120 + m, dtype=np.uint16) << 7), reps)
        w |= rng.integers(0, 128, w.size).astype(np.uint16)
    w = rng.permutation(w).astype(np.uint16)
    d, b = lwc.lwc_encode_dfloat11(w)
    h, (sym, _, _) = _blob_tables(b)
    from oracle import blob as B
    lengths = B.section(b, h["off_lengths"], 256)
    assert len(set(lengths[lengths > 0].tolist())) > 1
    assert _fixed_code_length(sym) == (0, False)
