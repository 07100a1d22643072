"""Oracle: the linear layer that consumes the decompressed weights.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The DFloat11 page ("Koniec z kompromisami! DFloat11 ratuje dokładność modeli
AI ...", section "Jak to działa w praktyce? Magia na poziomie GPU") has the
weights decompressed on the GPU during inference, just before the model uses
them, and measures the gain as token-generation throughput (section "Realne
korzyści, które zmieniają zasady gry"). What uses a decompressed matrix is the
transformer's linear layer; the pages do not write it out, so this module takes
its plain definition:

    y[m, r] = sum over c of W[r, c] * x[m, c]        (y = x @ W.T)

with W the tensor a blob decodes to, read as ``rows`` x ``cols`` row-major
(out_features x in_features, the layout the tensors are compressed in), and x
a batch of M activation rows, both BF16.

Readings where the pages are silent: values are those of the IEEE-754 binary32
numbers whose upper 16 bits are the BF16 pattern (BF16 is that format cut to a
7-bit mantissa); the sum is taken exactly enough in float64 that it serves as
the exact value for the tensor sizes tested (every product of two BF16 values
is exact in float64, and the error of the float64 sum is far below the float32
rounding bound below). A device result that accumulates in float32 in any
order is within ``float32_sum_bound`` of it (Higham, "Accuracy and Stability
of Numerical Algorithms", 2nd ed., section 4.2: |fl(sum) - sum| <= gamma_{n-1}
* sum |terms|, gamma_k = k u / (1 - k u), u = 2^-24), and a summation tree of
known height h within ``float32_tree_bound`` (gamma_h in place of
gamma_{n-1}), since the products themselves are exact in float32 (8 + 8
significant bits) unless they leave float32's exponent range.
"""
from __future__ import annotations

import numpy as np

from . import blob as B


def bf16_values(bits: np.ndarray) -> np.ndarray:
    """BF16 patterns to their values (float64), from the field definition:
    sign s (bit 15), exponent e (bits 14..7), fraction f (bits 6..0);
    e = 0: (-1)^s 2^-126 f/128; 0 < e < 255: (-1)^s 2^(e-127) (1 + f/128);
    e = 255: infinity (f = 0) or NaN."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.int64)
    s = (b >> 15) & 1
    e = (b >> 7) & 0xFF
    f = b & 0x7F
    sign = np.where(s == 1, -1.0, 1.0)
    normal = sign * np.ldexp(1.0 + f / 128.0, (e - 127).astype(np.int32))
    sub = sign * np.ldexp(f / 128.0, -126)
    special = np.where(f == 0, sign * np.inf, np.nan)
    return np.where(e == 0, sub, np.where(e == 255, special, normal))


def linear(w_bits: np.ndarray, x_bits: np.ndarray):
    """y = x W^T for BF16 patterns W (rows x cols) and x (M x cols).

    Returns (y, mag), both M x rows float64: the sums and the sums of the
    absolute products (the scale of the rounding bound)."""
    w = bf16_values(w_bits)
    x = bf16_values(x_bits)
    if w.ndim != 2 or x.ndim != 2 or w.shape[1] != x.shape[1]:
        raise ValueError("W must be rows x cols and x must be M x cols")
    y = x @ w.T
    mag = np.abs(x) @ np.abs(w).T
    return y, mag


def linear_rows(w_rows: np.ndarray, row_ids, x_bits: np.ndarray):
    """The outputs of the given rows only (for sampled checks of large
    tensors): w_rows holds those rows' BF16 patterns, one per row id."""
    y, mag = linear(np.asarray(w_rows).reshape(len(row_ids), -1), x_bits)
    return y, mag


def float32_tree_bound(mag: np.ndarray, height: int, unit_roundoff: float = 2.0 ** -24) -> np.ndarray:
    """Largest |float32 result - exact| for a sum of exact products taken
    along any summation tree in which no product passes through more than
    `height` float32 additions (or fused multiply-adds) on its way to the
    result: gamma_height * mag, u = 2^-24 (Higham, same section: each term
    picks up one factor (1 + delta), |delta| <= u, per addition on its path).
    `unit_roundoff` replaces u for additions that may round less well than
    round-to-nearest (2^-23 covers truncation to float32)."""
    u = unit_roundoff
    k = max(int(height), 0)
    gamma = k * u / (1.0 - k * u)
    return gamma * np.asarray(mag, dtype=np.float64)


def float32_sum_bound(mag: np.ndarray, cols: int) -> np.ndarray:
    """The order-free case: `cols` products in any order, gamma_{cols-1} * mag."""
    return float32_tree_bound(mag, cols - 1)


def from_blob(blob_bytes: np.ndarray, rows: int, cols: int, x_bits: np.ndarray):
    """Decode a blob of either codec with the oracle, then apply the layer."""
    from . import decode
    h = B.unpack_header(np.asarray(blob_bytes, np.uint8))
    if rows * cols != h["n"]:
        raise ValueError("rows * cols must equal the blob's weight count")
    w = decode(blob_bytes).reshape(rows, cols)
    return linear(w, x_bits)


def tile_order(w_bits: np.ndarray, tile_rows: int = 128, tile_cols: int = 64) -> np.ndarray:
    """The weights of a rows x cols matrix in tile order, flat: the matrix is
    cut into tile_rows x tile_cols tiles; tile (i, j) holds rows
    i*tile_rows .. (i+1)*tile_rows - 1 and columns j*tile_cols ..
    (j+1)*tile_cols - 1; tiles follow one another by i, then by j, and each
    tile is read row by row. This is the weight order the library's
    tensor-core product reads (a layout of this library; the pages do not
    fix one). Written tile by tile, as the definition reads."""
    w = np.asarray(w_bits)
    if w.ndim != 2:
        raise ValueError("expected a rows x cols matrix")
    rows, cols = w.shape
    if rows % tile_rows or cols % tile_cols:
        raise ValueError("rows and cols must be multiples of the tile size")
    pieces = []
    for i in range(rows // tile_rows):
        for j in range(cols // tile_cols):
            tile = w[i * tile_rows:(i + 1) * tile_rows, j * tile_cols:(j + 1) * tile_cols]
            pieces.append(tile.reshape(-1))
    return np.concatenate(pieces) if pieces else w.reshape(-1).copy()


def from_tile_order(flat: np.ndarray, rows: int, cols: int, tile_rows: int = 128, tile_cols: int = 64) -> np.ndarray:
    """The rows x cols matrix whose tile order is `flat` (inverse of
    tile_order), again tile by tile."""
    flat = np.asarray(flat).reshape(-1)
    if flat.size != rows * cols or rows % tile_rows or cols % tile_cols:
        raise ValueError("size and tile multiples do not match")
    w = np.empty((rows, cols), dtype=flat.dtype)
    k = 0
    for i in range(rows // tile_rows):
        for j in range(cols // tile_cols):
            n = tile_rows * tile_cols
            w[i * tile_rows:(i + 1) * tile_rows, j * tile_cols:(j + 1) * tile_cols] = \
                flat[k:k + n].reshape(tile_rows, tile_cols)
            k += n
    return w
