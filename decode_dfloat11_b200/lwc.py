"""ctypes binding of liblwc (include/lwc.h): argument marshalling only.

Every function keeps the C name. Host buffers are numpy arrays; device
buffers are passed as integer addresses (``tensor.data_ptr()``) or as torch
tensors, and streams as ``torch.cuda.Stream`` objects or raw handles. All
decoding happens in the library's CUDA kernels; there is no other path: if
liblwc.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblwc.so")

LWC_OK = 0
LWC_CODEC_DFLOAT11 = 1
LWC_CODEC_CODEBOOK = 2
LWC_ELEM_BF16 = 0
LWC_ELEM_FP32 = 1
LWC_ELEM_FP16 = 2
LWC_ERR_INVALID_ARG = 1
LWC_ERR_MISALIGNED = 2
LWC_ERR_CORRUPT = 3
LWC_ERR_UNSUPPORTED = 4
LWC_ERR_NOMEM = 5
LWC_ERR_CUDA = 6
LWC_DEVICE_BAD_COUNT = 1
LWC_DEVICE_BAD_CODE = 2
LWC_DEVICE_BAD_OFFSET = 4
LWC_DEVICE_TIMEOUT = 8

STATUS_NAMES = {0: "LWC_OK", 1: "LWC_ERR_INVALID_ARG", 2: "LWC_ERR_MISALIGNED", 3: "LWC_ERR_CORRUPT",
                4: "LWC_ERR_UNSUPPORTED", 5: "LWC_ERR_NOMEM", 6: "LWC_ERR_CUDA"}

# Every symbol include/lwc.h declares.
EXPORTED = (
    "lwc_encode_dfloat11", "lwc_encode_dfloat11_elements", "lwc_encode_codebook", "lwc_free", "lwc_desc_from_blob",
    "lwc_decode_dfloat11", "lwc_decode_codebook", "lwc_decode_dfloat11_checked",
    "lwc_decode_codebook_checked", "lwc_decode_dfloat11_batched", "lwc_decode_codebook_batched",
    "lwc_encode_device_workspace_bytes", "lwc_encode_dfloat11_device_plan",
    "lwc_encode_dfloat11_elements_device_plan", "lwc_encode_codebook_device_plan",
    "lwc_encode_device_write", "lwc_encode_dfloat11_device_noalloc", "lwc_linear_codebook",
    "lwc_linear_codebook_batched", "lwc_linear_dfloat11", "lwc_linear_dfloat11_batched",
    "lwc_tile_order", "lwc_gemm_dfloat11", "lwc_gemm_dfloat11_batched", "lwc_gemm_codebook",
    "lwc_gemm_codebook_batched",
    "lwc_selftest_bounded_wait", "lwc_status_string",
    "lwc_last_error", "lwc_version",
)


class LwcError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class lwc_desc(ctypes.Structure):
    _fields_ = [
        ("magic", ctypes.c_uint32), ("version", ctypes.c_uint32), ("codec", ctypes.c_uint32),
        ("flags", ctypes.c_uint32), ("n", ctypes.c_uint64), ("total_bytes", ctypes.c_uint64),
        ("chunk_bytes", ctypes.c_uint32), ("threads_per_block", ctypes.c_uint32),
        ("max_len", ctypes.c_uint32), ("n_tables", ctypes.c_uint32),
        ("n_chunks", ctypes.c_uint64), ("n_blocks", ctypes.c_uint64), ("total_bits", ctypes.c_uint64),
        ("max_block_count", ctypes.c_uint32), ("const_exp", ctypes.c_uint32),
        ("off_lengths", ctypes.c_uint64), ("off_lut", ctypes.c_uint64), ("off_gaps", ctypes.c_uint64),
        ("off_blkoff", ctypes.c_uint64), ("off_stream", ctypes.c_uint64), ("stream_bytes", ctypes.c_uint64),
        ("off_sm", ctypes.c_uint64),
        ("U", ctypes.c_uint32), ("k", ctypes.c_uint32), ("off_table", ctypes.c_uint64),
        ("off_packed", ctypes.c_uint64), ("packed_bytes", ctypes.c_uint64),
        ("elem", ctypes.c_uint32), ("reserved", ctypes.c_uint32), ("off_lo", ctypes.c_uint64),
        ("lo_bytes", ctypes.c_uint64), ("off_counts", ctypes.c_uint64),
    ]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}

    @property
    def bits_per_weight(self) -> float:
        return 8.0 * self.total_bytes / max(1, self.n)


class lwc_df11_params(ctypes.Structure):
    _fields_ = [("chunk_bytes", ctypes.c_uint32), ("threads_per_block", ctypes.c_uint32),
                ("max_len", ctypes.c_uint32), ("chunk_counts", ctypes.c_uint32)]


_lib = None
_P = ctypes.c_void_p
_u64 = ctypes.c_uint64


def load():
    """Load liblwc.so (built by decode_dfloat11_b200.build). Raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"liblwc.so not built ({LIB_PATH}); run python -m decode_dfloat11_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    D = ctypes.POINTER(lwc_desc)
    L.lwc_encode_dfloat11.argtypes = [_P, _u64, ctypes.POINTER(lwc_df11_params), D,
                                      ctypes.POINTER(_P), ctypes.POINTER(_u64)]
    L.lwc_encode_codebook.argtypes = [_P, _u64, D, ctypes.POINTER(_P), ctypes.POINTER(_u64)]
    L.lwc_encode_dfloat11_elements.argtypes = [_P, _u64, ctypes.c_uint32, ctypes.POINTER(lwc_df11_params), D,
                                               ctypes.POINTER(_P), ctypes.POINTER(_u64)]
    L.lwc_free.argtypes = [_P]
    L.lwc_free.restype = None
    L.lwc_desc_from_blob.argtypes = [_P, _u64, D]
    L.lwc_decode_dfloat11.argtypes = [D, _P, _P, _P]
    L.lwc_decode_codebook.argtypes = [D, _P, _P, _P]
    L.lwc_decode_dfloat11_checked.argtypes = [D, _P, _P, _P, _P]
    L.lwc_decode_codebook_checked.argtypes = [D, _P, _P, _P, _P]
    L.lwc_decode_dfloat11_batched.argtypes = [D, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.c_int, _P, _P]
    L.lwc_decode_codebook_batched.argtypes = [D, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.c_int, _P, _P]
    L.lwc_encode_device_workspace_bytes.argtypes = [_u64]
    L.lwc_encode_device_workspace_bytes.restype = _u64
    L.lwc_encode_dfloat11_device_plan.argtypes = [_P, _u64, ctypes.POINTER(lwc_df11_params), _P, _u64, D, _P]
    L.lwc_encode_codebook_device_plan.argtypes = [_P, _u64, _P, _u64, D, _P]
    L.lwc_encode_dfloat11_elements_device_plan.argtypes = [_P, _u64, ctypes.c_uint32, ctypes.POINTER(lwc_df11_params),
                                                           _P, _u64, D, _P]
    L.lwc_encode_device_write.argtypes = [_P, _u64, _P, _u64, _P, _u64, D, _P]
    L.lwc_encode_dfloat11_device_noalloc.argtypes = [_P, _u64, ctypes.POINTER(lwc_df11_params), _P, _u64, D, _P]
    for name in ("lwc_linear_codebook", "lwc_linear_dfloat11"):
        getattr(L, name).argtypes = [D, _P, _u64, _P, ctypes.c_int, _P, _P, _P]
        getattr(L, name).restype = ctypes.c_int
    for name in ("lwc_gemm_dfloat11", "lwc_gemm_codebook"):
        getattr(L, name).argtypes = [D, _P, _u64, _P, ctypes.c_int, _P, _P, _P]
        getattr(L, name).restype = ctypes.c_int
    L.lwc_tile_order.argtypes = [_P, _u64, _u64, _P, _P]
    L.lwc_tile_order.restype = ctypes.c_int
    for name in ("lwc_linear_codebook_batched", "lwc_linear_dfloat11_batched", "lwc_gemm_dfloat11_batched",
                 "lwc_gemm_codebook_batched"):
        getattr(L, name).argtypes = [D, ctypes.POINTER(_P), ctypes.POINTER(_u64), ctypes.POINTER(_P), ctypes.c_int,
                                     ctypes.POINTER(_P), ctypes.c_int, _P, _P]
        getattr(L, name).restype = ctypes.c_int
    L.lwc_selftest_bounded_wait.argtypes = [_P, ctypes.c_uint32, ctypes.c_int, _P]
    L.lwc_selftest_bounded_wait.restype = ctypes.c_int
    L.lwc_status_string.argtypes = [ctypes.c_int]
    L.lwc_status_string.restype = ctypes.c_char_p
    L.lwc_last_error.argtypes = []
    L.lwc_last_error.restype = ctypes.c_char_p
    L.lwc_version.argtypes = []
    for name in ("lwc_encode_dfloat11", "lwc_encode_dfloat11_elements", "lwc_encode_codebook", "lwc_desc_from_blob", "lwc_decode_dfloat11",
                 "lwc_decode_codebook", "lwc_decode_dfloat11_checked", "lwc_decode_codebook_checked",
                 "lwc_decode_dfloat11_batched", "lwc_decode_codebook_batched", "lwc_encode_dfloat11_device_plan",
                 "lwc_encode_codebook_device_plan", "lwc_encode_device_write",
                 "lwc_encode_dfloat11_elements_device_plan",
                 "lwc_encode_dfloat11_device_noalloc"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(status: int):
    if status != LWC_OK:
        raise LwcError(status, load().lwc_last_error().decode())


def _addr(x) -> int | None:
    """Device address of a torch tensor, or an integer address as given."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _take_blob(ptr: ctypes.c_void_p, nbytes: int) -> np.ndarray:
    L = load()
    try:
        out = np.empty(nbytes, np.uint8)
        if nbytes:
            ctypes.memmove(out.ctypes.data, ptr, nbytes)
        return out
    finally:
        L.lwc_free(ptr)


def _src(h_src) -> np.ndarray:
    a = np.ascontiguousarray(h_src)
    if a.dtype != np.uint16:
        a = a.view(np.uint16) if a.dtype.itemsize == 2 else a.astype(np.uint16)
    return a.reshape(-1)


def lwc_encode_dfloat11(h_src, chunk_bytes: int = 36, threads_per_block: int = 32,
                        max_len: int = 32, chunk_counts: bool = True) -> tuple[lwc_desc, np.ndarray]:
    """Encode host BF16 bit patterns (uint16 array); returns (desc, blob bytes).
    chunk_counts: store per-chunk code counts when they fit a byte (see lwc.h)."""
    src = _src(h_src)
    desc, ptr, nbytes = lwc_desc(), _P(), _u64()
    params = lwc_df11_params(chunk_bytes, threads_per_block, max_len, int(chunk_counts))
    _check(load().lwc_encode_dfloat11(src.ctypes.data, src.size, ctypes.byref(params), ctypes.byref(desc),
                                      ctypes.byref(ptr), ctypes.byref(nbytes)))
    return desc, _take_blob(ptr, nbytes.value)


def lwc_encode_dfloat11_elements(h_src, elem: int, chunk_bytes: int = 36, threads_per_block: int = 32,
                                 max_len: int = 32, chunk_counts: bool = True) -> tuple[lwc_desc, np.ndarray]:
    """DFloat11 encode of FP32 (uint32 / float32 array), FP16 or BF16 (16-bit) elements."""
    a = np.ascontiguousarray(h_src).reshape(-1)
    want = np.uint32 if elem == LWC_ELEM_FP32 else np.uint16
    if a.dtype != want:
        if a.dtype.itemsize != np.dtype(want).itemsize:
            raise ValueError(f"element type {elem} needs {np.dtype(want).itemsize}-byte elements")
        a = a.view(want)
    desc, ptr, nbytes = lwc_desc(), _P(), _u64()
    params = lwc_df11_params(chunk_bytes, threads_per_block, max_len, int(chunk_counts))
    _check(load().lwc_encode_dfloat11_elements(a.ctypes.data, a.size, elem, ctypes.byref(params), ctypes.byref(desc),
                                               ctypes.byref(ptr), ctypes.byref(nbytes)))
    return desc, _take_blob(ptr, nbytes.value)


def lwc_encode_codebook(h_src) -> tuple[lwc_desc, np.ndarray]:
    src = _src(h_src)
    desc, ptr, nbytes = lwc_desc(), _P(), _u64()
    _check(load().lwc_encode_codebook(src.ctypes.data, src.size, ctypes.byref(desc), ctypes.byref(ptr),
                                      ctypes.byref(nbytes)))
    return desc, _take_blob(ptr, nbytes.value)


def lwc_desc_from_blob(h_blob: np.ndarray) -> lwc_desc:
    b = np.ascontiguousarray(h_blob, dtype=np.uint8)
    desc = lwc_desc()
    _check(load().lwc_desc_from_blob(b.ctypes.data, b.size, ctypes.byref(desc)))
    return desc


def lwc_decode_dfloat11(desc: lwc_desc, d_in, d_out_bf16, stream=None) -> None:
    _check(load().lwc_decode_dfloat11(ctypes.byref(desc), _addr(d_in), _addr(d_out_bf16), _stream(stream)))


def lwc_decode_codebook(desc: lwc_desc, d_in, d_out_bf16, stream=None) -> None:
    _check(load().lwc_decode_codebook(ctypes.byref(desc), _addr(d_in), _addr(d_out_bf16), _stream(stream)))


def lwc_decode_dfloat11_checked(desc, d_in, d_out_bf16, d_status, stream=None) -> None:
    _check(load().lwc_decode_dfloat11_checked(ctypes.byref(desc), _addr(d_in), _addr(d_out_bf16),
                                              _addr(d_status), _stream(stream)))


def lwc_decode_codebook_checked(desc, d_in, d_out_bf16, d_status, stream=None) -> None:
    _check(load().lwc_decode_codebook_checked(ctypes.byref(desc), _addr(d_in), _addr(d_out_bf16),
                                              _addr(d_status), _stream(stream)))


class Batch:
    """Marshalled arguments of lwc_decode_dfloat11_batched, built once and
    reusable across calls (the layer loop decodes the same tensors again)."""

    def __init__(self, descs, d_ins, d_outs):
        n = len(descs)
        if not (len(d_ins) == len(d_outs) == n):
            raise ValueError("descs, d_ins and d_outs differ in length")
        self.count = n
        self.descs = (lwc_desc * max(1, n))(*descs)
        self.ins = (_P * max(1, n))(*[_addr(x) for x in d_ins])
        self.outs = (_P * max(1, n))(*[_addr(x) for x in d_outs])


def lwc_decode_dfloat11_batched(descs, d_ins=None, d_outs=None, d_status=None, stream=None) -> None:
    """Decode several DFloat11 tensors (e.g. one transformer layer) at once.
    ``descs`` may also be a prepared ``Batch`` (then d_ins/d_outs are unused)."""
    b = descs if isinstance(descs, Batch) else Batch(descs, d_ins, d_outs)
    _check(load().lwc_decode_dfloat11_batched(b.descs, b.ins, b.outs, b.count, _addr(d_status), _stream(stream)))


def lwc_decode_codebook_batched(descs, d_ins=None, d_outs=None, d_status=None, stream=None) -> None:
    """Decode several codebook tensors at once (one launch per index width)."""
    b = descs if isinstance(descs, Batch) else Batch(descs, d_ins, d_outs)
    _check(load().lwc_decode_codebook_batched(b.descs, b.ins, b.outs, b.count, _addr(d_status), _stream(stream)))


def lwc_linear_codebook(desc: lwc_desc, d_blob, cols: int, d_x, M: int, d_y, d_status=None, stream=None) -> None:
    """y = x W^T with W (n / cols x cols) decoded from a codebook blob in registers;
    x: M x cols BF16 (device), y: M x rows FP32 (device)."""
    _check(load().lwc_linear_codebook(ctypes.byref(desc), _addr(d_blob), cols, _addr(d_x), M, _addr(d_y),
                                      _addr(d_status), _stream(stream)))


def lwc_linear_dfloat11(desc: lwc_desc, d_blob, cols: int, d_x, M: int, d_y, d_status=None, stream=None) -> None:
    """As lwc_linear_codebook, for a DFloat11 blob of BF16 elements."""
    _check(load().lwc_linear_dfloat11(ctypes.byref(desc), _addr(d_blob), cols, _addr(d_x), M, _addr(d_y),
                                      _addr(d_status), _stream(stream)))


class LinearBatch:
    """Marshalled arguments of lwc_linear_*_batched, reusable across calls."""

    def __init__(self, descs, d_blobs, cols, d_xs, d_ys, M: int):
        n = len(descs)
        if not (len(d_blobs) == len(cols) == len(d_xs) == len(d_ys) == n):
            raise ValueError("argument lists differ in length")
        self.count = n
        self.M = M
        self.descs = (lwc_desc * max(1, n))(*descs)
        self.blobs = (_P * max(1, n))(*[_addr(x) for x in d_blobs])
        self.cols = (_u64 * max(1, n))(*cols)
        self.xs = (_P * max(1, n))(*[_addr(x) for x in d_xs])
        self.ys = (_P * max(1, n))(*[_addr(x) for x in d_ys])


def lwc_linear_codebook_batched(batch: LinearBatch, d_status=None, stream=None) -> None:
    b = batch
    _check(load().lwc_linear_codebook_batched(b.descs, b.blobs, b.cols, b.xs, b.M, b.ys, b.count, _addr(d_status),
                                              _stream(stream)))


def lwc_linear_dfloat11_batched(batch: LinearBatch, d_status=None, stream=None) -> None:
    b = batch
    _check(load().lwc_linear_dfloat11_batched(b.descs, b.blobs, b.cols, b.xs, b.M, b.ys, b.count, _addr(d_status),
                                              _stream(stream)))


def lwc_tile_order(d_src, rows: int, cols: int, d_dst, stream=None) -> None:
    """Write the 128 x 64 tile order of a rows x cols BF16 device matrix
    (the weight order lwc_gemm_dfloat11 reads) to d_dst."""
    _check(load().lwc_tile_order(_addr(d_src), rows, cols, _addr(d_dst), _stream(stream)))


def lwc_gemm_dfloat11(desc: lwc_desc, d_blob, cols: int, d_x, M: int, d_y, d_status=None, stream=None) -> None:
    """y = x W^T on the tensor cores, W decoded from a tile-order DFloat11
    blob into shared-memory operands; x: M x cols BF16, y: M x rows FP32
    (device), M = 1 .. 256."""
    _check(load().lwc_gemm_dfloat11(ctypes.byref(desc), _addr(d_blob), cols, _addr(d_x), M, _addr(d_y),
                                    _addr(d_status), _stream(stream)))


def lwc_gemm_dfloat11_batched(batch: LinearBatch, d_status=None, stream=None) -> None:
    """Several tile-order DFloat11 matrices (at most 8) in one launch."""
    b = batch
    _check(load().lwc_gemm_dfloat11_batched(b.descs, b.blobs, b.cols, b.xs, b.M, b.ys, b.count, _addr(d_status),
                                            _stream(stream)))


def lwc_gemm_codebook(desc: lwc_desc, d_blob, cols: int, d_x, M: int, d_y, d_status=None, stream=None) -> None:
    """As lwc_gemm_dfloat11, for a tile-order codebook blob."""
    _check(load().lwc_gemm_codebook(ctypes.byref(desc), _addr(d_blob), cols, _addr(d_x), M, _addr(d_y),
                                    _addr(d_status), _stream(stream)))


def lwc_gemm_codebook_batched(batch: LinearBatch, d_status=None, stream=None) -> None:
    """Several tile-order codebook matrices (at most 8, one index width) in one launch."""
    b = batch
    _check(load().lwc_gemm_codebook_batched(b.descs, b.blobs, b.cols, b.xs, b.M, b.ys, b.count, _addr(d_status),
                                            _stream(stream)))


def lwc_selftest_bounded_wait(d_status, polls: int, arrive: bool, stream=None) -> None:
    """Run the bounded-wait self-test kernel (see lwc.h)."""
    _check(load().lwc_selftest_bounded_wait(_addr(d_status), polls, int(bool(arrive)), _stream(stream)))


def lwc_encode_device_workspace_bytes(n: int) -> int:
    return load().lwc_encode_device_workspace_bytes(n)


def lwc_encode_dfloat11_device_plan(d_src, n: int, d_work, work_bytes: int, chunk_bytes: int = 36,
                                    threads_per_block: int = 32, max_len: int = 32, stream=None,
                                    chunk_counts: bool = True) -> lwc_desc:
    """Plan a DFloat11 blob for n device BF16 patterns; returns its descriptor."""
    desc = lwc_desc()
    params = lwc_df11_params(chunk_bytes, threads_per_block, max_len, int(chunk_counts))
    _check(load().lwc_encode_dfloat11_device_plan(_addr(d_src), n, ctypes.byref(params), _addr(d_work), work_bytes,
                                                  ctypes.byref(desc), _stream(stream)))
    return desc


def lwc_encode_dfloat11_elements_device_plan(d_src, n: int, elem: int, d_work, work_bytes: int, chunk_bytes: int = 36,
                                             threads_per_block: int = 32, max_len: int = 32,
                                             stream=None, chunk_counts: bool = True) -> lwc_desc:
    """Plan a DFloat11 blob of FP32 / FP16 / BF16 elements held on the device."""
    desc = lwc_desc()
    params = lwc_df11_params(chunk_bytes, threads_per_block, max_len, int(chunk_counts))
    _check(load().lwc_encode_dfloat11_elements_device_plan(_addr(d_src), n, elem, ctypes.byref(params), _addr(d_work),
                                                           work_bytes, ctypes.byref(desc), _stream(stream)))
    return desc


def lwc_encode_codebook_device_plan(d_src, n: int, d_work, work_bytes: int, stream=None) -> lwc_desc:
    desc = lwc_desc()
    _check(load().lwc_encode_codebook_device_plan(_addr(d_src), n, _addr(d_work), work_bytes, ctypes.byref(desc),
                                                  _stream(stream)))
    return desc


def lwc_encode_device_write(d_src, n: int, d_work, work_bytes: int, d_blob, blob_bytes: int,
                            stream=None) -> lwc_desc:
    """Write the planned blob into d_blob; returns the final descriptor."""
    desc = lwc_desc()
    _check(load().lwc_encode_device_write(_addr(d_src), n, _addr(d_work), work_bytes, _addr(d_blob), blob_bytes,
                                          ctypes.byref(desc), _stream(stream)))
    return desc


def lwc_encode_dfloat11_device_noalloc(d_src, n: int, d_blob, blob_bytes: int, chunk_bytes: int = 36,
                                       threads_per_block: int = 32, max_len: int = 32, stream=None,
                                       chunk_counts: bool = True) -> lwc_desc:
    """DFloat11 device encode without any device allocation (the library's
    own scratch array replaces the workspace); for callers that cannot call
    cudaMalloc. Returns the blob's descriptor."""
    desc = lwc_desc()
    params = lwc_df11_params(chunk_bytes, threads_per_block, max_len, int(chunk_counts))
    _check(load().lwc_encode_dfloat11_device_noalloc(_addr(d_src), n, ctypes.byref(params), _addr(d_blob),
                                                     blob_bytes, ctypes.byref(desc), _stream(stream)))
    return desc


def lwc_status_string(status: int) -> str:
    return load().lwc_status_string(status).decode()


def lwc_last_error() -> str:
    return load().lwc_last_error().decode()


def lwc_version() -> int:
    return load().lwc_version()
