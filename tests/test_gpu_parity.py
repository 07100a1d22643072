"""GPU decoders against the oracle, bit for bit, through the C ABI.

Small cases span many blocks/tiles with ragged tails; the full-size cases use
the workloads' own sizes (one Llama-3-8B layer, the 256M-weight codebook and
uniform-exponent stress tensors) with the launch configuration the benchmark
times. Every comparison is on 16-bit patterns (never float ==)."""
import numpy as np
import pytest
import torch

import synth
from decode_dfloat11_b200 import build as lwc_build
from decode_dfloat11_b200 import lwc
from oracle import blob as B
from oracle import codebook as ocb
from oracle import df11 as odf

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    lwc_build.build()
    return lwc.load()


def dev(blob: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(blob).to("cuda")


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def gpu_decode(desc, blob_dev, codec="df11", status=None):
    out = torch.empty(desc.n, dtype=torch.int16, device="cuda")
    st = torch.cuda.current_stream()
    if codec == "df11":
        lwc.lwc_decode_dfloat11_checked(desc, blob_dev, out, status, st)
    else:
        lwc.lwc_decode_codebook_checked(desc, blob_dev, out, status, st)
    torch.cuda.synchronize()
    return out


def small_inputs():
    yield "config1", synth.as_u16(synth.small_square(0))
    yield "uniform", synth.as_u16(synth.uniform_patterns(300_001, seed=1))
    yield "all_patterns", synth.as_u16(synth.all_patterns())
    yield "outliers", synth.as_u16(synth.normal_bf16((777_777,), seed=2, sigma=0.01, outlier_frac=1e-2))
    yield "narrow", synth.as_u16(synth.normal_bf16((500_000,), seed=3, sigma=1e-3))
    yield "single_exp", (np.arange(100_003, dtype=np.uint16) & 0x807F) | 0x3F00
    yield "zeros", np.zeros(4097, np.uint16)
    for n in (1, 2, 3, 15, 16, 17, 31, 33, 255, 257, 4095, 65537):
        yield f"n{n}", synth.as_u16(synth.normal_bf16((n,), seed=n, sigma=0.02))


@pytest.mark.parametrize("name,w", list(small_inputs()), ids=lambda x: x if isinstance(x, str) else "")
def test_df11_small(name, w):
    d, b = lwc.lwc_encode_dfloat11(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = host_u16(gpu_decode(d, dev(b), status=status))
    assert int(status.item()) == 0
    assert np.array_equal(got, odf.decode(b))
    assert np.array_equal(got, w)
    # the oracle's own blob decodes the same on the GPU
    ob = odf.encode(w)
    od = lwc.lwc_desc_from_blob(ob)
    assert np.array_equal(host_u16(gpu_decode(od, dev(ob))), w)


@pytest.mark.parametrize("chunk_bytes,tpb", [(8, 32), (12, 64), (20, 96), (36, 256), (64, 128), (36, 512),
                                             (36, 1024), (100, 32), (512, 32), (1024, 32)])
def test_df11_block_parameters(chunk_bytes, tpb):
    w = synth.as_u16(synth.normal_bf16((1_234_567,), seed=4, sigma=0.02, outlier_frac=1e-3))
    d, b = lwc.lwc_encode_dfloat11(w, chunk_bytes=chunk_bytes, threads_per_block=tpb)
    got = host_u16(gpu_decode(d, dev(b)))
    assert np.array_equal(got, odf.decode(b))
    ob = odf.encode(w, chunk_bytes=chunk_bytes, threads_per_block=tpb)
    assert np.array_equal(host_u16(gpu_decode(lwc.lwc_desc_from_blob(ob), dev(ob))), w)


def test_df11_long_codes():
    # Fibonacci counts make the Huffman tree a path (depth 31 for 32 symbols):
    # codes reach the length limit, the hierarchical tables go 4 levels deep
    # and the 12-bit fast tables miss for every rare exponent
    fib = [1, 1]
    while len(fib) < 32:
        fib.append(fib[-1] + fib[-2])
    w = np.repeat((np.arange(32, dtype=np.uint16) << 7) | 0x8011, np.array(fib))
    w = np.random.default_rng(0).permutation(w).astype(np.uint16)
    for limit, expect in ((32, 31), (24, 24), (16, 16)):
        d, b = lwc.lwc_encode_dfloat11(w, max_len=limit)
        assert d.max_len == expect
        assert np.array_equal(host_u16(gpu_decode(d, dev(b))), w)


@pytest.mark.parametrize("name,w", list(small_inputs()), ids=lambda x: x if isinstance(x, str) else "")
def test_codebook_small(name, w):
    d, b = lwc.lwc_encode_codebook(w)
    got = host_u16(gpu_decode(d, dev(b), codec="cb"))
    assert np.array_equal(got, ocb.decode(b))
    assert np.array_equal(got, w)


def test_codebook_identity_table_is_checked():
    """A table of all 65536 patterns is the identity (sorted distinct values),
    so the decoder copies the index stream; a blob whose table is not the
    identity is corrupt and is reported (LWC_DEVICE_BAD_CODE)."""
    w = synth.as_u16(synth.uniform_patterns(300_007, seed=11))
    w[:65536] = np.arange(65536, dtype=np.uint16)
    d, b = lwc.lwc_encode_codebook(w)
    assert d.U == 65536 and d.k == 16
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert np.array_equal(host_u16(gpu_decode(d, dev(b), codec="cb", status=status)), w)
    assert int(status.item()) == 0
    bad = b.copy()
    tab = bad[d.off_table:d.off_table + 2 * 65536].view(np.uint16)
    tab[[1000, 2000]] = tab[[2000, 1000]]    # no longer sorted: not a valid table
    gpu_decode(d, dev(bad), codec="cb", status=status)
    assert int(status.item()) & lwc.LWC_DEVICE_BAD_CODE


@pytest.mark.parametrize("U", [1, 2, 3, 5, 17, 200, 256, 600, 2000, 4096, 5000, 8192, 10000, 16384, 20000, 40000,
                               65536])
def test_codebook_every_width(U):
    n = 3 * 8192 + 77
    if U == 65536:
        w = synth.as_u16(synth.uniform_patterns(200_000, seed=U))
        w[:65536] = np.arange(65536, dtype=np.uint16)
    else:   # Zipf draws plus every table entry once, so U (and k) are exact
        draws = synth.as_u16(synth.codebook_stress(U, n, seed=U))
        table = synth.codebook_table(U, seed=U).numpy().astype(np.uint16)
        w = np.random.default_rng(U).permutation(np.concatenate([draws, table])).astype(np.uint16)
    d, b = lwc.lwc_encode_codebook(w)
    assert d.U == len(np.unique(w)) == U
    assert d.k == ocb.index_bits(U)
    got = host_u16(gpu_decode(d, dev(b), codec="cb"))
    assert np.array_equal(got, ocb.decode(b))
    assert np.array_equal(got, w)


def test_batched_mixed():
    tensors = [
        synth.as_u16(synth.normal_bf16((300_000,), seed=10, sigma=0.02)),
        (np.arange(5000, dtype=np.uint16) & 0x807F) | 0x3E80,           # single exponent
        np.zeros(0, np.uint16),
        synth.as_u16(synth.uniform_patterns(99_999, seed=11)),
        synth.as_u16(synth.normal_bf16((77,), seed=12, sigma=0.5)),
    ]
    params = [dict(), dict(), dict(), dict(chunk_bytes=12, threads_per_block=64), dict()]
    enc = [lwc.lwc_encode_dfloat11(w, **p) for w, p in zip(tensors, params)]
    blobs = [dev(b) for _, b in enc]
    outs = [torch.full((max(1, w.size),), 0x5555, dtype=torch.int16, device="cuda") for w in tensors]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lwc.lwc_decode_dfloat11_batched([d for d, _ in enc], blobs, outs, status, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for w, o in zip(tensors, outs):
        assert np.array_equal(host_u16(o)[:w.size], w)


def test_codebook_batched_mixed():
    tensors = [
        synth.as_u16(synth.codebook_stress(4096, 100_003, seed=20)),     # k = 12
        np.full(777, 0x3F80, np.uint16),                                # U = 1: k = 0
        np.zeros(0, np.uint16),
        synth.as_u16(synth.codebook_stress(300, 50_000, seed=21)),      # k = 9
        synth.as_u16(synth.codebook_stress(4000, 8_191, seed=22)),      # k = 12, one partial tile
        synth.as_u16(synth.uniform_patterns(70_000, seed=23)),          # k = 16
    ]
    enc = [lwc.lwc_encode_codebook(w) for w in tensors]
    blobs = [dev(b) for _, b in enc]
    outs = [torch.full((max(1, w.size),), 0x5555, dtype=torch.int16, device="cuda") for w in tensors]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lwc.lwc_decode_codebook_batched([d for d, _ in enc], blobs, outs, status, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for (d, b), w, o in zip(enc, tensors, outs):
        got = host_u16(o)[:w.size]
        assert np.array_equal(got, w)
        assert np.array_equal(got, ocb.decode(b))


def test_side_stream_and_reuse():
    w = synth.as_u16(synth.small_square(5))
    d, b = lwc.lwc_encode_dfloat11(w)
    bd = dev(b)
    s = torch.cuda.Stream()
    outs = [torch.empty(w.size, dtype=torch.int16, device="cuda") for _ in range(3)]
    with torch.cuda.stream(s):
        for o in outs:
            lwc.lwc_decode_dfloat11(d, bd, o, s)
    s.synchronize()
    for o in outs:
        assert np.array_equal(host_u16(o), w)


@pytest.mark.parametrize("tpb", [32, 256])   # the per-warp and the per-CTA kernel
def test_df11_corruption_is_contained(tpb):
    w = synth.as_u16(synth.small_square(6))
    d, b = lwc.lwc_encode_dfloat11(w, threads_per_block=tpb)
    rng = np.random.default_rng(0)
    guard = 4096
    cases = []
    x = b.copy()                                   # payload bit flips
    pos = d.off_stream + rng.integers(0, (d.total_bits + 7) // 8, 50)
    x[pos] ^= np.uint8(0x10)
    cases.append(x)
    x = b.copy()                                   # block offsets out of range
    x[d.off_blkoff + 8 * 3: d.off_blkoff + 8 * 4] = np.array([2 ** 40], np.uint64).view(np.uint8)
    cases.append(x)
    x = b.copy()                                   # every lookup entry invalid
    x[d.off_lut: d.off_lut + 512 * d.n_tables] = 0xFF
    cases.append(x)
    x = b.copy()                                   # gaps garbage
    x[d.off_gaps: d.off_gaps + d.n_blocks * d.threads_per_block] = rng.integers(0, 256, d.n_blocks * d.threads_per_block)
    cases.append(x)
    for i, x in enumerate(cases):
        xd = dev(x)
        out = torch.zeros(w.size + 2 * guard, dtype=torch.int16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        lwc.lwc_decode_dfloat11_checked(d, xd, out[guard:guard + w.size], status, torch.cuda.current_stream())
        torch.cuda.synchronize()
        got = host_u16(out)
        assert np.all(got[:guard] == 0) and np.all(got[guard + w.size:] == 0), i   # nothing outside
        assert int(status.item()) != 0 or not np.array_equal(got[guard:guard + w.size], w) or i == 0, i
        if i in (1, 2):
            assert int(status.item()) != 0, i


# ------------------------------------------------------------ fixed-length codes
#
# Flat exponent histograms over 2^L values give every code word length L; the
# counted decoder then reads a block's codes as back-to-back L-bit fields
# (the uniform-exponent stress tensor is L = 8). Chunk sizes whose bit count
# is not a multiple of L make codes straddle chunks (non-zero gaps).

@pytest.mark.parametrize("step", [1, 2])   # consecutive exponents (decoded without lookups) or not
@pytest.mark.parametrize("L", range(1, 9))
@pytest.mark.parametrize("chunk_bytes", [8, 20, 36])
def test_df11_fixed_length_codes(L, chunk_bytes, step):
    if step * ((1 << L) - 1) > 255:
        pytest.skip("2^L exponents with gaps do not fit in 8 bits")
    w = synth.as_u16(synth.equal_exponents(333_333 + 17 * L, L, seed=100 + L, step=step))
    d, b = lwc.lwc_encode_dfloat11(w, chunk_bytes=chunk_bytes)
    lengths = b[d.off_lengths:d.off_lengths + 256]
    assert set(lengths[lengths > 0].tolist()) == {L}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = host_u16(gpu_decode(d, dev(b), status=status))
    assert int(status.item()) == 0
    assert np.array_equal(got, odf.decode(b))
    assert np.array_equal(got, w)


@pytest.mark.parametrize("chunk_bytes", [8, 20, 36])
def test_df11_short_variable_length_codes(chunk_bytes):
    """Codes of at most 8 bits with more than one length (geometric exponent
    frequencies 2^7 : 2^6 : ... : 1 over 8 exponents, lengths 1..7): the kernel
    instance launched for short codes, on its block path."""
    rng = np.random.default_rng(chunk_bytes)
    counts = 1 << np.arange(7, -1, -1)
    e = np.repeat(np.arange(120, 128), counts * 2_000)
    w = ((e.astype(np.uint16) << 7) | rng.integers(0, 128, e.size).astype(np.uint16)
         | (rng.integers(0, 2, e.size).astype(np.uint16) << 15))
    w = rng.permutation(w).astype(np.uint16)
    d, b = lwc.lwc_encode_dfloat11(w, chunk_bytes=chunk_bytes)
    lengths = b[d.off_lengths:d.off_lengths + 256]
    assert d.max_len <= 8 and len(set(lengths[lengths > 0].tolist())) > 1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = host_u16(gpu_decode(d, dev(b), status=status))
    assert int(status.item()) == 0
    assert np.array_equal(got, odf.decode(b))
    assert np.array_equal(got, w)


def test_df11_fixed_length_batched_and_device_encoded():
    """Fixed- and variable-length tensors alternating in one launch (the CTA
    switches paths at each tensor boundary), encoded on the device."""
    from decode_dfloat11_b200.layers import encode_on_device
    ws = [synth.equal_exponents(200_003, 8, seed=61, device="cuda"),
          synth.normal_bf16((300_007,), seed=62, sigma=0.02, device="cuda"),
          synth.equal_exponents(150_001, 3, seed=63, step=3, device="cuda"),
          synth.equal_exponents(77_777, 6, seed=64, device="cuda"),
          synth.normal_bf16((1_001,), seed=65, sigma=0.02, device="cuda")]
    enc = [encode_on_device(w, "dfloat11") for w in ws]
    outs = [torch.empty(w.numel(), dtype=torch.int16, device="cuda") for w in ws]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lwc.lwc_decode_dfloat11_batched([d for d, _ in enc], [b for _, b in enc], outs, status,
                                    torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for w, (d, b), o in zip(ws, enc, outs):
        assert torch.equal(o, w.view(torch.int16).reshape(-1))
        assert np.array_equal(host_u16(o), odf.decode(b.cpu().numpy()))


def test_df11_fixed_length_corruption_is_contained():
    """A fixed-length tensor is decoded from the block offsets at the ends of
    each CTA's range and its stream: a first offset other than 0 or a last
    other than n is reported, an interior offset out of order either is
    reported (at a CTA boundary) or is not read, and nothing is written
    outside the output; damaged code words decode as the oracle decodes them;
    the gaps and counts are not read on this path."""
    w = synth.as_u16(synth.equal_exponents(500_000, 8, seed=9))
    d, b = lwc.lwc_encode_dfloat11(w)
    assert d.flags & 2
    guard = 4096
    cases = []
    for name, blk, v in (("first", 0, 64), ("last", d.n_blocks, 2 ** 40), ("interior", 3, 2 ** 40)):
        x = b.copy()
        x[d.off_blkoff + 8 * blk: d.off_blkoff + 8 * blk + 8] = np.array([v], np.uint64).view(np.uint8)
        cases.append((name, x))
    x = b.copy()                                   # payload bit flips: still valid code words
    pos = d.off_stream + np.random.default_rng(1).integers(0, (d.total_bits + 7) // 8, 50)
    x[pos] ^= np.uint8(0x10)
    cases.append(("payload", x))
    x = b.copy()                                   # gaps and counts garbage
    rng = np.random.default_rng(2)
    x[d.off_gaps: d.off_gaps + d.n_blocks * 32] = rng.integers(0, 256, d.n_blocks * 32)
    x[d.off_counts: d.off_counts + d.n_blocks * 32] = rng.integers(0, 256, d.n_blocks * 32)
    cases.append(("index", x))
    for name, x in cases:
        out = torch.zeros(w.size + 2 * guard, dtype=torch.int16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        lwc.lwc_decode_dfloat11_checked(d, dev(x), out[guard:guard + w.size], status, torch.cuda.current_stream())
        torch.cuda.synchronize()
        got = host_u16(out)
        assert np.all(got[:guard] == 0) and np.all(got[guard + w.size:] == 0), name   # nothing outside
        if name in ("first", "last"):
            assert int(status.item()) & lwc.LWC_DEVICE_BAD_OFFSET, name
        elif name == "interior":
            assert int(status.item()) & lwc.LWC_DEVICE_BAD_OFFSET or \
                (int(status.item()) == 0 and np.array_equal(got[guard:guard + w.size], w)), name
        elif name == "payload":
            assert int(status.item()) == 0 and np.array_equal(got[guard:guard + w.size], odf.decode(x)), name
        else:
            assert int(status.item()) == 0 and np.array_equal(got[guard:guard + w.size], w), name


# ------------------------------------------------------------ full-size configs

def test_llama3_8b_layer_full_size():
    """One Llama-3-8B layer (218,103,808 weights), DFloat11: per-tensor and
    layer-batched decodes, each compared with the oracle's decode of the same
    blob element by element."""
    tensors = [synth.as_u16(t) for _, t in synth.llama_layer_tensors(0)]
    enc = [lwc.lwc_encode_dfloat11(w) for w in tensors]
    blobs = [dev(b) for _, b in enc]
    outs = [torch.empty(w.size, dtype=torch.int16, device="cuda") for w in tensors]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lwc.lwc_decode_dfloat11_batched([d for d, _ in enc], blobs, outs, status, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for (d, b), w, o in zip(enc, tensors, outs):
        got = host_u16(o)
        assert np.array_equal(got, odf.decode(b))
        assert np.array_equal(got, w)
        o.zero_()
        lwc.lwc_decode_dfloat11(d, dev(b), o, torch.cuda.current_stream())
        torch.cuda.synchronize()
        assert np.array_equal(host_u16(o), w)
    bpw = 8.0 * sum(d.total_bytes for d, _ in enc) / sum(w.size for w in tensors)
    assert 10.0 < bpw < 11.5


@pytest.mark.parametrize("U", [256, 4096, 8192, 65536])
def test_codebook_stress_full_size(U):
    """256M weights from a U-entry table with Zipf(1.1) frequencies (the
    launch configuration bench.py times for the codebook stress figure)."""
    n = 1 << 28
    x = synth.codebook_stress(U, n, seed=40 + U, device="cuda")
    w = synth.as_u16(x)
    d, b = lwc.lwc_encode_codebook(w)
    assert d.k == {256: 8, 4096: 12, 8192: 13, 65536: 16}[U] or d.U < U
    out = gpu_decode(d, dev(b), codec="cb")
    assert torch.equal(out, x.view(torch.int16))
    # sampled windows, each read independently by the oracle
    rng = np.random.default_rng(U)
    got = host_u16(out)
    for i0 in list(rng.integers(0, n - 4096, 24)) + [n - 4096]:
        assert np.array_equal(got[i0:i0 + 4096], ocb.decode_range(b, int(i0), 4096))


def test_df11_uniform_exponents_full_size():
    """256M uniformly random patterns: all 256 exponents, 8-bit codes (an
    expansion to ~16 bits/weight), the decoder's worst table case."""
    n = 1 << 28
    x = synth.uniform_patterns(n, seed=77, device="cuda")
    w = synth.as_u16(x)
    d, b = lwc.lwc_encode_dfloat11(w)
    out = gpu_decode(d, dev(b))
    assert torch.equal(out, x.view(torch.int16))
    assert np.array_equal(host_u16(out), odf.decode(b))


@pytest.mark.parametrize("codec", ["codebook", "dfloat11"])
def test_fp16_patterns(codec):
    """FP16 weights as 16-bit patterns through both decoders, against the oracle."""
    w = synth.as_u16(synth.normal_fp16((1_000_003,), seed=12, sigma=0.02, outlier_frac=1e-3))
    if codec == "codebook":
        d, b = lwc.lwc_encode_codebook(w)
        ref = ocb.decode(b)
        got = host_u16(gpu_decode(d, dev(b), "cb"))
    else:
        d, b = lwc.lwc_encode_dfloat11(w)
        ref = odf.decode(b)
        got = host_u16(gpu_decode(d, dev(b), "df11"))
    assert np.array_equal(ref, w)
    assert np.array_equal(got, w)


# ------------------------------------------------------------ FP32 / FP16 elements

def element_cases():
    rng = np.random.default_rng(31)
    x32 = (rng.standard_normal(1_000_003).astype(np.float32) * 0.02).view(np.uint32)
    yield "fp32_normal", B.ELEM_FP32, x32
    special = np.array([0, 0x80000000, 0x7F800000, 0xFF800000, 0x7FC00001, 0xFFFFFFFF, 1, 0x807FFFFF], np.uint32)
    yield "fp32_random", B.ELEM_FP32, np.concatenate(
        [special, rng.integers(0, 2 ** 32, 300_001, dtype=np.uint64).astype(np.uint32)])
    yield "fp16_normal", B.ELEM_FP16, synth.as_u16(synth.normal_fp16((1_000_003,), seed=13, sigma=0.02,
                                                                      outlier_frac=1e-3))
    yield "fp16_all", B.ELEM_FP16, np.arange(65536, dtype=np.uint16)
    yield "fp16_single_exp", B.ELEM_FP16, ((np.arange(70_001) & 0x83FF) | (13 << 10)).astype(np.uint16)
    yield "fp32_single_exp", B.ELEM_FP32, ((np.arange(70_001, dtype=np.uint32) * 2654435761) & 0x807FFFFF) | (120 << 23)
    for n in (1, 15, 16, 17, 33, 4097):
        yield f"fp16_n{n}", B.ELEM_FP16, rng.integers(0, 65536, n, dtype=np.uint64).astype(np.uint16)
        yield f"fp32_n{n}", B.ELEM_FP32, rng.integers(0, 2 ** 32, n, dtype=np.uint64).astype(np.uint32)


def gpu_decode_elements(d, blob_dev, elem, n):
    out = torch.zeros(n, dtype=torch.int32 if elem == B.ELEM_FP32 else torch.int16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lwc.lwc_decode_dfloat11_checked(d, blob_dev, out, status, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = out.cpu().numpy()
    return got.view(np.uint32) if elem == B.ELEM_FP32 else got.view(np.uint16)


@pytest.mark.parametrize("tpb", [32, 256])   # the per-warp and the per-CTA kernel
@pytest.mark.parametrize("name,elem,x", list(element_cases()), ids=lambda v: v if isinstance(v, str) else "")
def test_df11_elements(name, elem, x, tpb):
    d, b = lwc.lwc_encode_dfloat11_elements(x, elem, threads_per_block=tpb)
    ref = odf.decode_elements(b)
    assert np.array_equal(ref, x)
    assert np.array_equal(gpu_decode_elements(d, dev(b), elem, x.size), x)


def test_df11_elements_mixed_batch():
    """BF16, FP32 and FP16 tensors in one batched call (one launch per element type)."""
    rng = np.random.default_rng(32)
    xs = [(B.ELEM_BF16, synth.as_u16(synth.normal_bf16((500_001,), seed=40, sigma=0.02))),
          (B.ELEM_FP32, (rng.standard_normal(300_007).astype(np.float32) * 0.03).view(np.uint32)),
          (B.ELEM_FP16, synth.as_u16(synth.normal_fp16((400_009,), seed=41, sigma=0.01))),
          (B.ELEM_FP32, (rng.standard_normal(12_345).astype(np.float32)).view(np.uint32))]
    enc = [lwc.lwc_encode_dfloat11_elements(x, e) for e, x in xs]
    blobs = [dev(b) for _, b in enc]
    outs = [torch.zeros(x.size, dtype=torch.int32 if e == B.ELEM_FP32 else torch.int16, device="cuda")
            for e, x in xs]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lwc.lwc_decode_dfloat11_batched([d for d, _ in enc], blobs, outs, status, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for (e, x), o in zip(xs, outs):
        got = o.cpu().numpy()
        assert np.array_equal(got.view(np.uint32) if e == B.ELEM_FP32 else got.view(np.uint16), x), e


def test_df11_fp32_full_size():
    """An FP32 matrix of the Llama-3-8B gate shape (58,720,256 weights, 235 MB out)."""
    x = synth.normal_bf16((14336, 4096), seed=42, sigma=0.02).float()   # FP32 values with BF16 precision ...
    x = x + torch.randn(x.shape, generator=torch.Generator().manual_seed(43)) * 1e-5   # ... plus low bits
    xh = x.numpy().view(np.uint32).reshape(-1)
    d, b = lwc.lwc_encode_dfloat11_elements(xh, B.ELEM_FP32)
    got = gpu_decode_elements(d, dev(b), B.ELEM_FP32, xh.size)
    assert np.array_equal(got, xh)
    assert 8.0 * d.total_bytes / d.n < 28.0


@pytest.mark.parametrize("elem", [B.ELEM_FP32, B.ELEM_FP16])
def test_df11_wide_form_elements(elem):
    """A launch of at least 512 M weights takes the counted decoder's wide form
    (one 32-warp CTA per SM): 2^29 + 12,345 FP32 / FP16 elements encoded on the
    device, decoded, compared with the input, and sampled block ranges of the
    coded 16-bit patterns compared with the oracle's block-range decode."""
    from decode_dfloat11_b200.layers import encode_on_device
    n = (1 << 29) + 12_345
    g = torch.Generator(device="cuda").manual_seed(90 + elem)
    x = torch.randn(n, generator=g, device="cuda") * 0.02
    x = x if elem == B.ELEM_FP32 else x.to(torch.float16)
    d, blob = encode_on_device(x, "dfloat11")
    assert d.elem == elem and d.flags & 2 and d.max_len > 8
    out = torch.empty(n, dtype=torch.int32 if elem == B.ELEM_FP32 else torch.int16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lwc.lwc_decode_dfloat11_checked(d, blob, out, status, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(out, x.view(torch.int32 if elem == B.ELEM_FP32 else torch.int16))
    hb = blob.cpu().numpy()
    xs = x.view(torch.int32 if elem == B.ELEM_FP32 else torch.int16).cpu().numpy()
    xs = xs.view(np.uint32) if elem == B.ELEM_FP32 else xs.view(np.uint16)
    blkoff = B.section(hb, d.off_blkoff, 8 * (d.n_blocks + 1), np.uint64)
    for b0 in (0, d.n_blocks // 3, d.n_blocks - 3):
        v = odf.decode_blocks(hb, b0, b0 + 3)
        i0, i1 = int(blkoff[b0]), int(blkoff[b0 + 3])
        assert np.array_equal(v, odf.split_elements(xs[i0:i1], elem)[0]), b0
