"""Host side of liblwc, no GPU needed: the library loads and exports every
symbol include/lwc.h declares; its encoders' blobs decode in the oracle (and
pass the oracle's re-derivation of gaps, block offsets and lookup tables);
it parses the oracle's blobs; and it rejects damaged headers and bad
arguments before touching a device."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth
from conftest import ROOT
from decode_dfloat11_b200 import build as lwc_build
from decode_dfloat11_b200 import lwc
from oracle import blob as B
from oracle import codebook as ocb
from oracle import df11 as odf


@pytest.fixture(scope="module", autouse=True)
def built():
    lwc_build.build()
    return lwc.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "lwc.h")).read()
    return sorted(set(re.findall(r"LWC_API\s+[\w\s\*]+?\b(lwc_\w+)\s*\(", text)))


def test_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 12
    L = lwc.load()
    for name in names:
        assert hasattr(L, name), name
    assert set(names) == set(lwc.EXPORTED)
    assert lwc.lwc_version() == 10000
    assert lwc.lwc_status_string(3) == "corrupt blob or descriptor"


def df11_inputs():
    yield "config1", synth.as_u16(synth.small_square(0))
    yield "uniform", synth.as_u16(synth.uniform_patterns(300_001, seed=1))
    yield "all_patterns", synth.as_u16(synth.all_patterns())
    yield "outliers", synth.as_u16(synth.normal_bf16((777_777,), seed=2, sigma=0.01, outlier_frac=1e-2))
    yield "single_exp", (np.arange(10_000, dtype=np.uint16) & 0x807F) | 0x3F00
    yield "zeros", np.zeros(123, np.uint16)
    yield "empty", np.zeros(0, np.uint16)
    for n in (1, 2, 3, 7, 31, 33, 255, 257):
        yield f"n{n}", synth.as_u16(synth.uniform_patterns(n, seed=n))


@pytest.mark.parametrize("name,w", list(df11_inputs()), ids=lambda x: x if isinstance(x, str) else "")
def test_library_df11_blob_decodes_in_oracle(name, w):
    d, b = lwc.lwc_encode_dfloat11(w)
    assert d.total_bytes == b.size and d.n == w.size
    assert np.array_equal(odf.decode(b), w)
    assert odf.check_index(b) == []
    assert lwc.lwc_desc_from_blob(b).as_dict() == d.as_dict()


@pytest.mark.parametrize("chunk_bytes,tpb", [(8, 32), (12, 64), (36, 256), (64, 128), (36, 1024), (100, 512)])
def test_library_df11_parameters(chunk_bytes, tpb):
    w = synth.as_u16(synth.normal_bf16((250_007,), seed=5, sigma=0.02, outlier_frac=1e-3))
    d, b = lwc.lwc_encode_dfloat11(w, chunk_bytes=chunk_bytes, threads_per_block=tpb)
    assert (d.chunk_bytes, d.threads_per_block) == (chunk_bytes, tpb)
    assert np.array_equal(odf.decode(b), w)
    assert odf.check_index(b) == []


def test_library_code_is_optimal_like_the_oracle():
    # both encoders build an optimal code: same total bits, possibly other codewords
    for seed in range(3):
        w = synth.as_u16(synth.normal_bf16((400_000,), seed=seed, sigma_range=(0.005, 0.04),
                                           outlier_frac=1e-3))
        d, _ = lwc.lwc_encode_dfloat11(w)
        oh = B.unpack_header(odf.encode(w))
        assert d.total_bits == oh["total_bits"]


def test_library_length_limit():
    # Fibonacci counts: a Huffman tree 39 deep; the library must limit it
    fib = [1, 1]
    while len(fib) < 40:
        fib.append(fib[-1] + fib[-2])
    counts = np.array(fib[:40], np.int64) // 1000 + 1
    w = np.repeat((np.arange(40, dtype=np.uint16) << 7) | 0x8005, counts)
    w = np.random.default_rng(0).permutation(w).astype(np.uint16)
    for limit in (32, 16, 12):
        d, b = lwc.lwc_encode_dfloat11(w, max_len=limit)
        assert d.max_len <= limit
        assert np.array_equal(odf.decode(b), w)
        assert odf.check_index(b) == []


@pytest.mark.parametrize("U", [1, 2, 3, 255, 256, 257, 4096, 8192, 65536])
def test_library_codebook_blob_decodes_in_oracle(U):
    n = 70_001 if U < 65536 else 300_000
    w = synth.as_u16(synth.codebook_stress(U, n, seed=U)) if U < 65536 else \
        synth.as_u16(synth.uniform_patterns(n, seed=9))
    d, b = lwc.lwc_encode_codebook(w)
    assert d.U == len(np.unique(w)) and d.k == ocb.index_bits(d.U)
    assert np.array_equal(ocb.decode(b), w)
    # same layout rule, same table, same packing: the bytes agree with the oracle's
    assert np.array_equal(b, ocb.encode(w))


def test_library_parses_oracle_blobs():
    w = synth.as_u16(synth.small_square(3))
    ob = odf.encode(w, chunk_bytes=20, threads_per_block=96)
    d = lwc.lwc_desc_from_blob(ob)
    h = B.unpack_header(ob)
    for key, val in h.items():
        if key in ("header_bytes",):
            continue
        assert getattr(d, key) == val, key
    oc = ocb.encode(w)
    dc = lwc.lwc_desc_from_blob(oc)
    assert (dc.U, dc.k, dc.n) == (B.unpack_header(oc)["U"], B.unpack_header(oc)["k"], w.size)


def corrupt(blob, off, fmt, value):
    b = blob.copy()
    b[off:off + np.dtype(fmt).itemsize] = np.array([value], fmt).view(np.uint8)
    return b


def test_damaged_headers_are_rejected():
    w = synth.as_u16(synth.small_square(1))
    _, b = lwc.lwc_encode_dfloat11(w)
    h = B.unpack_header(b)
    bad = [
        corrupt(b, 0, "<u4", 0x12345678),                 # magic
        corrupt(b, 4, "<u2", 2),                          # version
        corrupt(b, 16, "<u8", h["total_bytes"] + 16),     # size mismatch
        corrupt(b, 32, "<u4", 30),                        # chunk_bytes not a multiple of 4
        corrupt(b, 36, "<u4", 48),                        # threads_per_block not a multiple of 32
        corrupt(b, 40, "<u4", 40),                        # max_len beyond the format
        corrupt(b, 48, "<u8", h["n_chunks"] + 1),         # chunk count
        corrupt(b, 56, "<u8", h["n_blocks"] + 1),         # block count
        corrupt(b, 64, "<u8", 8),                         # total_bits below n
        corrupt(b, 72, "<u4", 0),                         # max_block_count
        corrupt(b, 112, "<u8", h["total_bytes"] - 16),    # stream outside the blob
        corrupt(b, 128, "<u8", 8),                        # misaligned section
    ]
    for i, x in enumerate(bad):
        with pytest.raises(lwc.LwcError) as e:
            lwc.lwc_desc_from_blob(x)
        assert e.value.status == 3, i
    with pytest.raises(lwc.LwcError):
        lwc.lwc_desc_from_blob(b[:100])
    _, c = lwc.lwc_encode_codebook(w)
    for x in (corrupt(c, 36, "<u4", 11), corrupt(c, 32, "<u4", 100_000), corrupt(c, 56, "<u8", 16)):
        with pytest.raises(lwc.LwcError) as e:
            lwc.lwc_desc_from_blob(x)
        assert e.value.status == 3


def test_decoders_validate_before_any_device_call():
    w = synth.as_u16(synth.small_square(2))
    d, _ = lwc.lwc_encode_dfloat11(w)
    dc, _ = lwc.lwc_encode_codebook(w)
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_decode_dfloat11(d, 0x1008, 0x2000)          # misaligned input
    assert e.value.status == 2
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_decode_codebook(dc, 0x1000, 0x2002)         # misaligned output
    assert e.value.status == 2
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_decode_dfloat11(dc, 0x1000, 0x2000)         # wrong codec
    assert e.value.status == 1
    bad = lwc.lwc_desc.from_buffer_copy(d)
    bad.n_blocks += 1
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_decode_dfloat11(bad, 0x1000, 0x2000)
    assert e.value.status == 3
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_decode_dfloat11_batched([d, d], [0x1000, None], [0x2000, 0x3000])
    assert e.value.status == 1
    # empty tensors need no device at all
    d0, _ = lwc.lwc_encode_dfloat11(np.zeros(0, np.uint16))
    lwc.lwc_decode_dfloat11(d0, None, None)
    c0, _ = lwc.lwc_encode_codebook(np.zeros(0, np.uint16))
    lwc.lwc_decode_codebook(c0, None, None)


def test_linear_layer_validates_before_any_device_call():
    # y = x W^T entry points: every argument error is reported before a CUDA call
    w = synth.as_u16(synth.normal_bf16((64 * 48,), seed=3, sigma=0.02))
    d, _ = lwc.lwc_encode_dfloat11(w)
    dc, _ = lwc.lwc_encode_codebook(w)
    for desc, fn in ((d, lwc.lwc_linear_dfloat11), (dc, lwc.lwc_linear_codebook)):
        for M in (0, 9, -1):                                           # 1..8 activation rows
            with pytest.raises(lwc.LwcError) as e:
                fn(desc, 0x1000, 48, 0x2000, M, 0x3000)
            assert e.value.status == 1 and "M must be" in str(e.value)
        for cols in (0, 47, 64 * 48 + 1, 1 << 31):                    # must divide n, < 2^31
            with pytest.raises(lwc.LwcError) as e:
                fn(desc, 0x1000, cols, 0x2000, 1, 0x3000)
            assert e.value.status == 1
        for args in ((0x1008, 0x2000, 0x3000), (0x1000, 0x2008, 0x3000), (0x1000, 0x2000, 0x3002)):
            with pytest.raises(lwc.LwcError) as e:                     # blob, x 16-byte; y 4-byte aligned
                fn(desc, args[0], 48, args[1], 1, args[2])
            assert e.value.status == 2
        with pytest.raises(lwc.LwcError) as e:
            fn(desc, None, 48, 0x2000, 1, 0x3000)
        assert e.value.status == 1
    with pytest.raises(lwc.LwcError) as e:                             # wrong codec
        lwc.lwc_linear_dfloat11(dc, 0x1000, 48, 0x2000, 1, 0x3000)
    assert e.value.status == 1
    # DFloat11 blobs the fused layer does not take
    d256, _ = lwc.lwc_encode_dfloat11(w, threads_per_block=256)
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_linear_dfloat11(d256, 0x1000, 48, 0x2000, 1, 0x3000)
    assert e.value.status == 4 and "32 chunks" in str(e.value)
    x32 = np.arange(64 * 48, dtype=np.uint32) * 2654435761 % (1 << 31)
    d32, _ = lwc.lwc_encode_dfloat11_elements(x32.astype(np.uint32), lwc.LWC_ELEM_FP32)
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_linear_dfloat11(d32, 0x1000, 48, 0x2000, 1, 0x3000)
    assert e.value.status == 4 and "BF16" in str(e.value)
    # batched: argument lists must agree; empty tensors need no device
    with pytest.raises(ValueError):
        lwc.LinearBatch([d, d], [0x1000], [48, 48], [0x2000, 0x2000], [0x3000, 0x3000], 1)
    d0, _ = lwc.lwc_encode_dfloat11(np.zeros(0, np.uint16))
    c0, _ = lwc.lwc_encode_codebook(np.zeros(0, np.uint16))
    lwc.lwc_linear_dfloat11_batched(lwc.LinearBatch([d0], [None], [16], [None], [None], 2))
    lwc.lwc_linear_codebook_batched(lwc.LinearBatch([c0, c0], [None, None], [1, 7], [None, None], [None, None], 8))


def test_wait_selftest_validates_before_any_device_call():
    for args in ((None, 64, False), (0x1002, 64, False), (0x1000, 0, True), (0x1000, (1 << 24) + 1, True)):
        with pytest.raises(lwc.LwcError) as e:
            lwc.lwc_selftest_bounded_wait(*args)
        assert e.value.status == 1


def test_fused_linear_helper_checks_shapes_before_the_library():
    import torch
    from decode_dfloat11_b200.layers import fused_linear
    w = synth.as_u16(synth.normal_bf16((16 * 32,), seed=4, sigma=0.02))
    d, b = lwc.lwc_encode_codebook(w)
    ok = torch.zeros((2, 32), dtype=torch.bfloat16)
    bad_cases = [
        dict(shape=(16, 32), x=torch.zeros((2, 31), dtype=torch.bfloat16)),          # wrong cols
        dict(shape=(16, 32), x=torch.zeros((2, 32), dtype=torch.float16)),           # not BF16
        dict(shape=(16, 32), x=torch.zeros(32, dtype=torch.bfloat16)),               # not M x cols
        dict(shape=(512,), x=ok),                                                    # W not a matrix
        dict(shape=(16, 32), x=ok, out=torch.empty((2, 15), dtype=torch.float32)),   # wrong out shape
        dict(shape=(16, 32), x=ok, out=torch.empty((2, 16), dtype=torch.float64)),   # wrong out dtype
    ]
    for case in bad_cases:
        with pytest.raises(ValueError):
            fused_linear(d, b, case["shape"], case["x"], "codebook", out=case.get("out"))
    with pytest.raises(ValueError):
        fused_linear(d, b, (16, 32), ok, "huffman")


def test_header_is_plain_c(tmp_path):
    # the boundary is a C ABI: include/lwc.h must compile as strict C99 (and C++)
    import shutil
    import subprocess
    src = tmp_path / "use_lwc.c"
    src.write_text('#include "lwc.h"\nint main(void) { lwc_desc d; (void)d; return (int)LWC_OK; }\n')
    for cc, std in (("gcc", "-std=c99"), ("g++", "-std=c++17")):
        if shutil.which(cc) is None:
            pytest.skip(f"{cc} not installed")
        lang = ["-x", "c++"] if cc == "g++" else []
        r = subprocess.run([cc, std, "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only", "-I",
                            os.path.join(ROOT, "include"), *lang, str(src)], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_encoder_rejects_bad_arguments():
    w = np.zeros(10, np.uint16)
    for kw in (dict(chunk_bytes=6), dict(chunk_bytes=10), dict(threads_per_block=48),
               dict(threads_per_block=2048), dict(max_len=8), dict(max_len=33)):
        with pytest.raises(lwc.LwcError) as e:
            lwc.lwc_encode_dfloat11(w, **kw)
        assert e.value.status == 1
    L = lwc.load()
    desc = lwc.lwc_desc()
    assert L.lwc_encode_dfloat11(None, 5, None, ctypes.byref(desc), None, None) == 1


def test_encode_many_matches_sequential():
    from decode_dfloat11_b200.layers import encode_many
    arrays = [synth.as_u16(synth.normal_bf16((50_000 + 17 * i,), seed=30 + i, sigma=0.02, outlier_frac=1e-3))
              for i in range(6)]
    for codec, fn in (("dfloat11", lwc.lwc_encode_dfloat11), ("codebook", lwc.lwc_encode_codebook)):
        par = encode_many(arrays, codec, workers=4)
        for (d, b), a in zip(par, arrays):
            d2, b2 = fn(a)
            assert np.array_equal(b, b2) and d.as_dict() == d2.as_dict()
    with pytest.raises(ValueError):
        encode_many(arrays, "zstd")


def test_device_encoder_validates_before_any_device_call():
    L = lwc.load()
    n = 100_000
    need = lwc.lwc_encode_device_workspace_bytes(n)
    # the workspace holds the tile arrays (DFloat11) or the 65536-entry index map (codebook)
    tiles = (n + 4095) // 4096
    assert need >= 256 + 8192 + max(2 * 65536, 12 * tiles)
    assert lwc.lwc_encode_device_workspace_bytes(1 << 30) >= 12 * ((1 << 30) // 4096)
    assert need % 256 == 0
    cases = [
        (lambda: lwc.lwc_encode_dfloat11_device_plan(0x1000, n, None, need), 1),          # no workspace
        (lambda: lwc.lwc_encode_dfloat11_device_plan(0x1000, n, 0x2000, need - 1), 1),    # too small
        (lambda: lwc.lwc_encode_dfloat11_device_plan(0x1008, n, 0x2000, need), 2),        # misaligned source
        (lambda: lwc.lwc_encode_dfloat11_device_plan(0x1000, n, 0x2010, need), 2),        # misaligned workspace
        (lambda: lwc.lwc_encode_dfloat11_device_plan(None, n, 0x2000, need), 1),          # no source
        (lambda: lwc.lwc_encode_dfloat11_device_plan(0x1000, n, 0x2000, need, chunk_bytes=10), 1),
        (lambda: lwc.lwc_encode_dfloat11_device_plan(0x1000, n, 0x2000, need, max_len=40), 1),
        (lambda: lwc.lwc_encode_codebook_device_plan(0x1000, 1 << 37, 0x2000, 1 << 62), 4),  # above the limit
        (lambda: lwc.lwc_encode_device_write(0x1000, n, 0x2000, need, None, 1 << 20), 1),  # no blob
        (lambda: lwc.lwc_encode_device_write(0x1000, n, 0x2000, need, 0x9008, 1 << 20), 2),  # misaligned blob
    ]
    for i, (call, status) in enumerate(cases):
        with pytest.raises(lwc.LwcError) as e:
            call()
        assert e.value.status == status, (i, str(e.value))
    desc = lwc.lwc_desc()
    assert L.lwc_encode_codebook_device_plan(0x1000, n, 0x2000, need, None, None) == 1
    assert L.lwc_encode_device_write(0x1000, n, 0x2000, need, 0x3000, 1 << 20, None, None) == 1
    del desc


def test_fp16_weights_through_both_codecs():
    """FP16 weights (the codebook pages' proof of concept used FP16): both
    codecs take any 16-bit patterns, so FP16 round-trips bit for bit. The
    codebook's index width follows the tensor's distinct FP16 values; the
    DFloat11 split is BF16-specific, so on FP16 patterns it is lossless but
    compresses less (its 'exponent' byte straddles FP16's exponent and
    mantissa)."""
    w = synth.as_u16(synth.normal_fp16((300_007,), seed=11, sigma=0.02, outlier_frac=1e-3))
    d, b = lwc.lwc_encode_codebook(w)
    assert d.U == len(np.unique(w)) and d.k == ocb.index_bits(d.U)
    assert np.array_equal(ocb.decode(b), w)
    assert np.array_equal(b, ocb.encode(w))
    d2, b2 = lwc.lwc_encode_dfloat11(w)
    assert np.array_equal(odf.decode(b2), w)
    assert odf.check_index(b2) == []
    assert d2.bits_per_weight > 11.0   # far less skewed 'exponent' byte than BF16's


def elements_inputs():
    rng = np.random.default_rng(21)
    x32 = (rng.standard_normal(200_003).astype(np.float32) * 0.02).view(np.uint32)
    yield "fp32_normal", B.ELEM_FP32, x32
    special = np.array([0x00000000, 0x80000000, 0x7F800000, 0xFF800000, 0x7FC00001, 0xFFFFFFFF,
                        0x00000001, 0x807FFFFF, 0x3F800000], np.uint32)
    yield "fp32_special", B.ELEM_FP32, np.concatenate([special, rng.integers(0, 2 ** 32, 70_001,
                                                                             dtype=np.uint64).astype(np.uint32)])
    yield "fp16_normal", B.ELEM_FP16, synth.as_u16(synth.normal_fp16((300_007,), seed=12, sigma=0.02,
                                                                      outlier_frac=1e-3))
    yield "fp16_all", B.ELEM_FP16, np.arange(65536, dtype=np.uint16)
    for n in (1, 2, 5, 15, 16, 17, 33):
        yield f"fp16_n{n}", B.ELEM_FP16, rng.integers(0, 65536, n, dtype=np.uint64).astype(np.uint16)
        yield f"fp32_n{n}", B.ELEM_FP32, rng.integers(0, 2 ** 32, n, dtype=np.uint64).astype(np.uint32)
    yield "fp16_single_exp", B.ELEM_FP16, ((np.arange(10_000) & 0x83FF) | (13 << 10)).astype(np.uint16)
    yield "fp32_empty", B.ELEM_FP32, np.zeros(0, np.uint32)


@pytest.mark.parametrize("name,elem,x", list(elements_inputs()), ids=lambda v: v if isinstance(v, str) else "")
def test_library_element_blobs_decode_in_oracle(name, elem, x):
    d, b = lwc.lwc_encode_dfloat11_elements(x, elem)
    assert d.elem == elem and d.total_bytes == b.size and d.n == x.size
    assert np.array_equal(odf.decode_elements(b), x)
    assert odf.check_index(b) == []
    assert lwc.lwc_desc_from_blob(b).as_dict() == d.as_dict()
    # the oracle's own blob parses in the library with the same element fields
    ob = odf.encode_elements(x, elem, threads_per_block=32)
    od = lwc.lwc_desc_from_blob(ob)
    assert (od.elem, od.lo_bytes) == (elem, B.unpack_header(ob)["lo_bytes"])


def test_element_encoder_arguments():
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_encode_dfloat11_elements(np.zeros(4, np.uint16), 7)
    assert e.value.status == 1
    # BF16 through the element entry point is the BF16 encoder
    w = synth.as_u16(synth.small_square(4))
    assert np.array_equal(lwc.lwc_encode_dfloat11_elements(w, B.ELEM_BF16)[1], lwc.lwc_encode_dfloat11(w)[1])
    # a damaged element field or short low-mantissa section is rejected
    d, b = lwc.lwc_encode_dfloat11_elements(np.arange(1000, dtype=np.uint32) * 77777, B.ELEM_FP32)
    for x in (corrupt(b, 136, "<u4", 3), corrupt(b, 152, "<u8", 16)):
        with pytest.raises(lwc.LwcError) as e:
            lwc.lwc_desc_from_blob(x)
        assert e.value.status == 3


def test_resident_model_needs_two_buffers():
    # the pipelined layer loop decodes layer L + 1 while layer L is in use:
    # a single output buffer would let the two overlap, so it is refused
    from decode_dfloat11_b200.layers import ResidentModel
    with pytest.raises(ValueError):
        ResidentModel("dfloat11", "cpu", slots=1)
    with pytest.raises(ValueError):
        ResidentModel("dfloat11", "cpu", slots=0)
    assert ResidentModel("codebook", "cpu", slots=2).slots == 2


def test_tensor_core_product_rejects_bad_arguments_before_any_device_work():
    """lwc_gemm_dfloat11 checks its arguments on the host before it touches
    the device: these calls fail the same way with or without a GPU (the
    device pointers are never dereferenced)."""
    from oracle import linear as OL
    w = synth.as_u16(synth.normal_bf16((256, 128), seed=1, sigma=0.02)).reshape(256, 128)
    d, _ = lwc.lwc_encode_dfloat11(OL.tile_order(w), chunk_bytes=20)
    fake = ctypes.c_void_p(1 << 40)          # 16-byte aligned, never read
    def call(desc, cols, M, blob=fake, x=fake, y=fake):
        L = lwc.load()
        return L.lwc_gemm_dfloat11(ctypes.byref(desc), blob, cols, x, M, y, None, None)
    assert call(d, 128, 0) == lwc.LWC_ERR_INVALID_ARG
    assert call(d, 128, 257) == lwc.LWC_ERR_INVALID_ARG
    assert call(d, 96, 4) == lwc.LWC_ERR_INVALID_ARG           # cols not a multiple of 64
    assert call(d, 256 * 128, 4) == lwc.LWC_ERR_INVALID_ARG    # rows = 1, not a multiple of 128
    assert call(d, 128, 4, blob=None) == lwc.LWC_ERR_INVALID_ARG
    assert call(d, 128, 4, x=ctypes.c_void_p((1 << 40) + 2)) == lwc.LWC_ERR_MISALIGNED
    for kw in ({"chunk_counts": False}, {"threads_per_block": 64}):
        d2, _ = lwc.lwc_encode_dfloat11(OL.tile_order(w), **kw)
        assert call(d2, 128, 4) == lwc.LWC_ERR_UNSUPPORTED
    d3, _ = lwc.lwc_encode_dfloat11(np.full(256 * 128, 0x3F80, np.uint16))   # one exponent value
    assert call(d3, 128, 4) == lwc.LWC_ERR_UNSUPPORTED
    dc, _ = lwc.lwc_encode_codebook(OL.tile_order(w))
    assert call(dc, 128, 4) != lwc.LWC_OK                      # not a DFloat11 blob
    # the tile order itself
    L = lwc.load()
    assert L.lwc_tile_order(fake, 100, 128, ctypes.c_void_p((1 << 40) + 4096), None) == lwc.LWC_ERR_INVALID_ARG
    assert L.lwc_tile_order(fake, 256, 96, ctypes.c_void_p((1 << 40) + 4096), None) == lwc.LWC_ERR_INVALID_ARG
    assert L.lwc_tile_order(fake, 256, 128, fake, None) == lwc.LWC_ERR_INVALID_ARG
    assert L.lwc_tile_order(fake, 0, 128, ctypes.c_void_p((1 << 40) + 4096), None) == lwc.LWC_OK
