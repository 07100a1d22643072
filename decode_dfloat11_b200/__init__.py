"""Lossless BF16 weight decompression on NVIDIA B200 (sm_100a).

The product is the C library ``liblwc.so`` (C ABI in ``include/lwc.h``):
host encoders for the DFloat11-style exponent-Huffman codec and the codebook
codec, and CUDA decoders that expand compressed tensors back to bit-exact BF16
in GPU memory. ``decode_dfloat11_b200.lwc`` is its ctypes binding and
``decode_dfloat11_b200.build`` compiles it.
"""
from . import lwc  # noqa: F401

__all__ = ["lwc"]
