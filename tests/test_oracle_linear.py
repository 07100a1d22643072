"""Pins of the linear-layer oracle (oracle/linear.py) against facts that do not
come from it: the IEEE-754 field values of BF16 patterns (hand-derived, and
numpy's own float32 conversion of the pattern's upper half), a hand-derived
worked example under tests/golden/, closed forms (all-ones sums, one-hot
columns), exact rational arithmetic on small cases, and real float32
summation for the rounding bound."""
import math
from fractions import Fraction

import numpy as np
import pytest

import synth
from conftest import load_golden
from oracle import codebook, df11
from oracle import linear as OL

G = load_golden("linear_worked_example.json")


def hexes(rows):
    return np.array([[int(v, 16) for v in r] for r in rows], np.uint16)


def expected_value(v):
    table = {"2^-126": 2.0 ** -126, "2^-133": 2.0 ** -133, "255 * 2^120": 255.0 * 2.0 ** 120,
             "-0": -0.0, "inf": math.inf, "-inf": -math.inf, "nan": math.nan}
    return table[v] if isinstance(v, str) else float(v)


def test_bf16_field_values():
    for h, v in G["patterns"]:
        got = float(OL.bf16_values(np.array([int(h, 16)], np.uint16))[0])
        want = expected_value(v)
        if math.isnan(want):
            assert math.isnan(got), h
        else:
            assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), h


def test_bf16_values_match_float32_upper_half_on_every_pattern():
    bits = np.arange(65536, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        lib = (bits << 16).view(np.float32).astype(np.float64)
    got = OL.bf16_values(bits.astype(np.uint16))
    assert np.array_equal(got, lib, equal_nan=True)
    num = ~np.isnan(lib)   # a NaN's sign carries no value
    assert np.array_equal(np.signbit(got[num]), np.signbit(lib[num]))


def test_golden_rectangular_example():
    y, mag = OL.linear(hexes(G["rect"]["W_hex"]), hexes(G["rect"]["x_hex"]))
    assert np.array_equal(y, np.array(G["rect"]["y"]))
    assert np.array_equal(mag, np.array(G["rect"]["mag"]))


def test_golden_square_example_catches_a_transpose():
    y, _ = OL.linear(hexes(G["square"]["W_hex"]), hexes(G["square"]["x_hex"]))
    assert np.array_equal(y, np.array(G["square"]["y"]))


def test_ones_closed_form():
    rows, cols = 5, 200
    w = np.full((rows, cols), 0x3F80, np.uint16)                  # 1.0
    # x[m, c] = c + 1 (integers <= 256 are exact in BF16)
    vals = np.arange(1, cols + 1, dtype=np.float32)
    x = (vals.view(np.uint32) >> 16).astype(np.uint16)[None, :].repeat(3, 0)
    y, mag = OL.linear(w, x)
    assert np.all(y == cols * (cols + 1) / 2) and np.all(mag == y)


@pytest.mark.parametrize("c", [0, 1, 6, 36])
def test_one_hot_selects_a_column(c):
    w = synth.as_u16(synth.normal_bf16((9, 37), seed=3, sigma=0.02)).reshape(9, 37)
    x = np.zeros((2, 37), np.uint16)
    x[0, c] = 0x3F80          # 1.0
    x[1, c] = 0xC000          # -2.0
    y, _ = OL.linear(w, x)
    col = OL.bf16_values(w[:, c])
    assert np.array_equal(y[0], col) and np.array_equal(y[1], -2.0 * col)


@pytest.mark.parametrize("seed", range(4))
def test_exact_rational_sums(seed):
    rng = np.random.default_rng(seed)
    rows, cols, M = 4, 7, 3
    w = synth.as_u16(synth.normal_bf16((rows * cols,), seed=10 + seed, sigma=0.02)).reshape(rows, cols)
    x = synth.as_u16(synth.normal_bf16((M * cols,), seed=20 + seed, sigma=1.0)).reshape(M, cols)
    x[rng.integers(0, M), rng.integers(0, cols)] = 0x8000   # a -0 activation
    y, mag = OL.linear(w, x)

    def frac(h):   # the pattern's exact value as a fraction (finite patterns only)
        f32 = np.array([int(h) << 16], np.uint32).view(np.float32)[0]
        return Fraction(float(f32))
    for m in range(M):
        for r in range(rows):
            exact = sum((frac(w[r, c]) * frac(x[m, c]) for c in range(cols)), Fraction(0))
            a = sum((abs(frac(w[r, c]) * frac(x[m, c])) for c in range(cols)), Fraction(0))
            assert abs(Fraction(y[m, r]) - exact) <= Fraction(2) ** -50 * a
            assert mag[m, r] == float(a) or abs(Fraction(mag[m, r]) - a) <= Fraction(2) ** -50 * a


def test_float32_bound_closed_form_and_real_float32_sums():
    assert OL.float32_sum_bound(np.array([1.0]), 1)[0] == 0.0
    k = 4096
    g = k * 2.0 ** -24 / (1 - k * 2.0 ** -24)
    assert OL.float32_sum_bound(np.array([2.0]), k + 1)[0] == 2.0 * g
    assert OL.float32_tree_bound(np.array([2.0]), k)[0] == 2.0 * g
    rng = np.random.default_rng(5)
    cols = 4096
    w = synth.as_u16(synth.normal_bf16((cols,), seed=6, sigma=0.02)).reshape(1, cols)
    x = synth.as_u16(synth.normal_bf16((cols,), seed=7, sigma=1.0)).reshape(1, cols)
    y, mag = OL.linear(w, x)
    prods = (OL.bf16_values(w[0]) * OL.bf16_values(x[0])).astype(np.float32)
    assert np.array_equal(prods.astype(np.float64), OL.bf16_values(w[0]) * OL.bf16_values(x[0]))  # exact
    # a left-to-right float32 sum in a random order stays inside the order-free bound
    order = rng.permutation(cols)
    acc = np.float32(0)
    for v in prods[order]:
        acc = np.float32(acc + v)
    assert abs(float(acc) - y[0, 0]) <= OL.float32_sum_bound(mag, cols)[0, 0]
    # pairwise float32 summation (height 12) stays inside the height-12 bound
    level = prods[order]
    height = 0
    while level.size > 1:
        level = (level[0::2] + level[1::2]).astype(np.float32)
        height += 1
    assert height == 12
    tree = OL.float32_tree_bound(mag, height)[0, 0]
    assert abs(float(level[0]) - y[0, 0]) <= tree
    # and losing the largest product is far outside it
    big = int(np.argmax(np.abs(prods)))
    assert abs(float(level[0]) - float(prods[big]) - y[0, 0]) > 100 * tree


def test_from_blob_both_codecs():
    rows, cols = 33, 48
    w = synth.as_u16(synth.normal_bf16((rows * cols,), seed=30, sigma=0.02, outlier_frac=1e-2))
    x = synth.as_u16(synth.normal_bf16((2 * cols,), seed=31, sigma=1.0)).reshape(2, cols)
    want, _ = OL.linear(w.reshape(rows, cols), x)
    for blob in (df11.encode(w), codebook.encode(w)):
        y, _ = OL.from_blob(blob, rows, cols, x)
        assert np.array_equal(y, want)
    with pytest.raises(ValueError):
        OL.from_blob(df11.encode(w), rows, cols + 1, x)


def test_golden_tile_order():
    """The tile order of a hand-worked 4 x 6 example (2 x 3 tiles), and back."""
    g = G["tile_order"]
    w = np.arange(g["rows"] * g["cols"], dtype=np.uint16).reshape(g["rows"], g["cols"])
    got = OL.tile_order(w, g["tile_rows"], g["tile_cols"])
    assert got.tolist() == g["tile_order"]
    back = OL.from_tile_order(np.array(g["tile_order"], np.uint16), g["rows"], g["cols"], g["tile_rows"], g["tile_cols"])
    assert np.array_equal(back, w)


def test_tile_order_is_a_permutation_with_closed_form_positions():
    """Every weight appears once, and weight (r, c) of a 256 x 192 matrix
    lands where its tile and its place in the tile say: tiles before it
    (all earlier tile rows, then earlier tiles of its own tile row) hold
    8192 weights each, then r % 128 full tile rows of 64, then c % 64."""
    rows, cols = 256, 192
    w = np.arange(rows * cols, dtype=np.uint32).reshape(rows, cols)
    t = OL.tile_order(w)
    assert np.array_equal(np.sort(t), np.arange(rows * cols))
    for r, c in [(0, 0), (0, 63), (0, 64), (1, 0), (127, 191), (128, 0), (200, 100), (255, 191)]:
        tiles_before = (r // 128) * (cols // 64) + c // 64
        pos = tiles_before * 8192 + (r % 128) * 64 + c % 64
        assert t[pos] == w[r, c]
    assert np.array_equal(OL.from_tile_order(t, rows, cols), w)


def test_tile_order_whole_matrix_tile_is_row_major():
    w = np.arange(128 * 64, dtype=np.uint16).reshape(128, 64)
    assert np.array_equal(OL.tile_order(w), w.reshape(-1))
    with pytest.raises(ValueError):
        OL.tile_order(np.zeros((100, 64), np.uint16))
