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
