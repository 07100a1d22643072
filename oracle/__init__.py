"""Oracle for the lossless BF16 weight codecs — TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct CPU implementation of what the decode path
computes: the DFloat11-style exponent-Huffman codec (``oracle.df11``, with
the code construction in ``oracle.huffman``) and the codebook codec
(``oracle.codebook``), over the container in ``oracle.blob``; and the linear
layer that consumes a decompressed matrix (``oracle.linear``, float64, with
the float32 rounding bounds a device result is held to). The per-weight
loops are plain C (``native.c``, one bit at a time); the rest is Python.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package. It shares no code with the CUDA
library in ``decode_dfloat11_b200`` and imports nothing from it; the two meet
only through the blob format.

Pins (checked by ``tests/test_oracle_*.py`` against facts that do not come
from the oracle itself): decode is the identity on every 16-bit pattern
(round trip, all 65536 patterns, brute force over tiny tensors); the Huffman
code is complete and prefix-free (integer Kraft sum), optimal (brute force
over all length vectors on small alphabets, with and without a length
limit) and within one bit of the exponent entropy; the canonical codes and
bit order match hand-derived worked examples under ``tests/golden/``; the
codebook width is ceil(log2 U) and its table is the sorted set of distinct
patterns (checked against a brute-force count); BF16 values follow the
IEEE-754 fields (hand-derived values, numpy's float32 view on all 65536
patterns), and the linear layer matches a hand-derived worked example,
closed forms, one-hot columns and exact rational sums. The exact bytes of a
stream are pinned only through those worked examples: the pages print no
encoded example of their own.
"""
from . import blob, codebook, df11, huffman, linear
from ._native import build

__all__ = ["blob", "codebook", "df11", "huffman", "linear", "build", "decode"]


def decode(blob_bytes):
    """Decode a blob of either codec to uint16 BF16 patterns."""
    import numpy as np
    h = blob.unpack_header(np.asarray(blob_bytes, np.uint8))
    if h["codec"] == blob.CODEC_DFLOAT11:
        return df11.decode(blob_bytes)
    return codebook.decode(blob_bytes)
