"""Device encoders through the C ABI: the blob built on the GPU must be the
host encoder's blob byte for byte (same code, same layout, same padding), and
it must decode back to the source, on the GPU and in the oracle.

Inputs span ragged sizes (tails inside a 16-weight group, a 4096-weight
tile, a 1024-weight packing group), single-exponent and single-value tensors,
every 16-bit pattern, long codes, all DFloat11 parameter shapes the format
allows, and full Llama-3-8B layer shapes."""
import numpy as np
import pytest
import torch

import synth
from decode_dfloat11_b200 import build as lwc_build
from decode_dfloat11_b200 import lwc
from decode_dfloat11_b200.layers import ResidentModel, encode_on_device
from oracle import codebook as ocb
from oracle import df11 as odf

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    lwc_build.build()
    return lwc.load()


def on_gpu(w: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(w.view(np.int16).copy()).to("cuda")


def host_bytes(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def decode(desc, blob, codec):
    out = torch.empty(desc.n, dtype=torch.int16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fn = lwc.lwc_decode_dfloat11_checked if codec == "dfloat11" else lwc.lwc_decode_codebook_checked
    fn(desc, blob, out, status, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out.cpu().numpy().view(np.uint16)


def inputs():
    yield "config1", synth.as_u16(synth.small_square(0))
    yield "uniform", synth.as_u16(synth.uniform_patterns(300_001, seed=1))
    yield "all_patterns", synth.as_u16(synth.all_patterns())
    yield "outliers", synth.as_u16(synth.normal_bf16((777_777,), seed=2, sigma=0.01, outlier_frac=1e-2))
    yield "single_exp", (np.arange(100_003, dtype=np.uint16) & 0x807F) | 0x3F00
    yield "zeros", np.zeros(4097, np.uint16)
    for n in (1, 2, 7, 15, 16, 17, 1023, 1025, 4095, 4096, 4097, 65537):
        yield f"n{n}", synth.as_u16(synth.normal_bf16((n,), seed=n, sigma=0.02))


CASES = list(inputs())


@pytest.mark.parametrize("codec", ["dfloat11", "codebook"])
@pytest.mark.parametrize("name,w", CASES, ids=lambda x: x if isinstance(x, str) else "")
def test_device_blob_equals_host_blob(name, w, codec):
    host_fn = lwc.lwc_encode_dfloat11 if codec == "dfloat11" else lwc.lwc_encode_codebook
    hd, hb = host_fn(w)
    dd, db = encode_on_device(on_gpu(w), codec)
    assert dd.as_dict() == hd.as_dict()
    dbh = host_bytes(db)
    assert np.array_equal(dbh, hb)
    # the device-made blob itself, checked by the oracle: its indexes (gaps,
    # block offsets, chunk counts, tables) re-derived from a sequential
    # decode, and its decode
    if codec == "dfloat11":
        assert odf.check_index(dbh) == []
        assert np.array_equal(odf.decode(dbh), w)
    else:
        assert np.array_equal(ocb.decode(dbh), w)
    if w.size:
        assert np.array_equal(decode(dd, db, codec), w)


@pytest.mark.parametrize("chunk_bytes,tpb,max_len", [(8, 32, 32), (12, 64, 32), (36, 256, 16), (64, 128, 12),
                                                     (36, 1024, 32), (100, 512, 32), (1024, 32, 32)])
def test_device_df11_parameters(chunk_bytes, tpb, max_len):
    w = synth.as_u16(synth.normal_bf16((250_007,), seed=5, sigma=0.02, outlier_frac=1e-3))
    params = dict(chunk_bytes=chunk_bytes, threads_per_block=tpb, max_len=max_len)
    hd, hb = lwc.lwc_encode_dfloat11(w, **params)
    dd, db = encode_on_device(on_gpu(w), "dfloat11", **params)
    assert dd.as_dict() == hd.as_dict()
    assert np.array_equal(host_bytes(db), hb)
    assert np.array_equal(odf.decode(hb), w)


def test_device_df11_long_codes():
    # Fibonacci exponent counts give a 31-deep Huffman tree; limits 32/24/16 apply
    fib = [1, 1]
    while len(fib) < 32:
        fib.append(fib[-1] + fib[-2])
    w = np.repeat((np.arange(32, dtype=np.uint16) << 7) | 0x8005, fib)
    w = np.random.default_rng(0).permutation(w).astype(np.uint16)
    for limit in (32, 24, 16):
        hd, hb = lwc.lwc_encode_dfloat11(w, max_len=limit)
        dd, db = encode_on_device(on_gpu(w), "dfloat11", max_len=limit)
        assert np.array_equal(host_bytes(db), hb) and dd.as_dict() == hd.as_dict()
        assert np.array_equal(decode(dd, db, "dfloat11"), w)


@pytest.mark.parametrize("U", [2, 3, 255, 256, 257, 4096, 8192, 65536])
def test_device_codebook_widths(U):
    n = 700_001
    w = synth.as_u16(synth.codebook_stress(U, n, seed=U)) if U < 65536 else \
        synth.as_u16(synth.uniform_patterns(n, seed=9))
    hd, hb = lwc.lwc_encode_codebook(w)
    dd, db = encode_on_device(on_gpu(w), "codebook")
    assert dd.as_dict() == hd.as_dict()
    assert np.array_equal(host_bytes(db), hb)
    assert np.array_equal(ocb.decode(hb), w)


def test_workspace_reuse_across_tensors_and_codecs():
    work = torch.empty(lwc.lwc_encode_device_workspace_bytes(400_000), dtype=torch.uint8, device="cuda")
    for i, n in enumerate((400_000, 17, 123_457, 4096)):
        w = synth.as_u16(synth.normal_bf16((n,), seed=40 + i, sigma=0.03, outlier_frac=1e-3))
        for codec, fn in (("dfloat11", lwc.lwc_encode_dfloat11), ("codebook", lwc.lwc_encode_codebook)):
            work.fill_(0xAB)   # leftovers of earlier calls must not matter
            dd, db = encode_on_device(on_gpu(w), codec, workspace=work)
            hd, hb = fn(w)
            assert np.array_equal(host_bytes(db), hb), (codec, n)


@pytest.mark.parametrize("which", ["q", "k", "o", "gate", "down"])
def test_device_encode_llama3_8b_layer_tensors(which):
    spec = [s for s in synth.LLAMA3_8B_LAYER if s[0] == which]
    (j, t), = synth.llama_layer_tensors(3, spec, (0.01, 0.04), 0, device="cuda")
    w = synth.as_u16(t)
    for codec, fn in (("dfloat11", lwc.lwc_encode_dfloat11), ("codebook", lwc.lwc_encode_codebook)):
        dd, db = encode_on_device(t, codec)
        hd, hb = fn(w)
        assert dd.as_dict() == hd.as_dict()
        assert np.array_equal(host_bytes(db), hb), (codec, j)
        out = torch.empty(dd.n, dtype=torch.int16, device="cuda")
        f = lwc.lwc_decode_dfloat11 if codec == "dfloat11" else lwc.lwc_decode_codebook
        f(dd, db, out, torch.cuda.current_stream())
        torch.cuda.synchronize()
        assert torch.equal(out, t.reshape(-1).view(torch.int16))


def test_resident_model_from_device_tensors():
    shapes = [(3072, 1024), (1024, 3072), (17, 33)]
    tensors = [synth.normal_bf16(s, 900 + j, sigma=0.02, outlier_frac=1e-3, device="cuda")
               for j, s in enumerate(shapes)]
    for codec in ("dfloat11", "codebook"):
        m = ResidentModel(codec, "cuda")
        m.add_layer_from_device("layer0", tensors)
        m.finalize()
        m.decode(0, 0, torch.cuda.current_stream())
        torch.cuda.synchronize()
        for v, t in zip(m.views(0, 0), tensors):
            assert torch.equal(v.view(torch.int16), t.view(torch.int16)), codec


def test_device_encoder_errors():
    w = synth.as_u16(synth.normal_bf16((10_000,), seed=7, sigma=0.02))
    src = on_gpu(w)
    n = w.size
    need = lwc.lwc_encode_device_workspace_bytes(n)
    work = torch.zeros(need, dtype=torch.uint8, device="cuda")
    blob = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    # no plan in the workspace
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_encode_device_write(src, n, work, need, blob, blob.numel())
    assert e.value.status == 1
    # workspace too small, misaligned source
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_encode_dfloat11_device_plan(src, n, work, need - 256)
    assert e.value.status == 1
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_encode_dfloat11_device_plan(src.data_ptr() + 2, n - 1, work, need)
    assert e.value.status == 2
    # blob buffer too small
    d = lwc.lwc_encode_dfloat11_device_plan(src, n, work, need)
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_encode_device_write(src, n, work, need, blob, d.total_bytes - 16)
    assert e.value.status == 1
    # different n than planned
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_encode_device_write(src, n - 1, work, need, blob, blob.numel())
    assert e.value.status == 1
    # the source changed between plan and write: detected, and nothing is
    # written outside the planned blob (the canary after it survives)
    other = on_gpu(synth.as_u16(synth.normal_bf16((n,), seed=8, sigma=0.5)))
    for codec_plan in (lwc.lwc_encode_dfloat11_device_plan, lwc.lwc_encode_codebook_device_plan):
        d = codec_plan(src, n, work, need)
        blob.fill_(0x5A)
        with pytest.raises(lwc.LwcError) as e:
            lwc.lwc_encode_device_write(other, n, work, need, blob, d.total_bytes)
        assert e.value.status == 1
        torch.cuda.synchronize()
        assert bool((blob[d.total_bytes:] == 0x5A).all())
    # and the plan still works with the right source
    d = lwc.lwc_encode_dfloat11_device_plan(src, n, work, need)
    d2 = lwc.lwc_encode_device_write(src, n, work, need, blob, blob.numel())
    assert np.array_equal(host_bytes(blob[:d2.total_bytes]), lwc.lwc_encode_dfloat11(w)[1])


def element_sources():
    rng = np.random.default_rng(51)
    x32 = (rng.standard_normal(300_007).astype(np.float32) * 0.02).view(np.uint32)
    yield "fp32_normal", 1, x32
    yield "fp32_random", 1, rng.integers(0, 2 ** 32, 70_001, dtype=np.uint64).astype(np.uint32)
    yield "fp16_normal", 2, synth.as_u16(synth.normal_fp16((300_007,), seed=52, sigma=0.02, outlier_frac=1e-3))
    yield "fp16_all", 2, np.arange(65536, dtype=np.uint16)
    yield "fp16_single_exp", 2, ((np.arange(10_001) & 0x83FF) | (13 << 10)).astype(np.uint16)
    for n in (1, 15, 16, 17, 4097):
        yield f"fp32_n{n}", 1, rng.integers(0, 2 ** 32, n, dtype=np.uint64).astype(np.uint32)
        yield f"fp16_n{n}", 2, rng.integers(0, 65536, n, dtype=np.uint64).astype(np.uint16)


@pytest.mark.parametrize("name,elem,x", list(element_sources()), ids=lambda v: v if isinstance(v, str) else "")
def test_device_element_blob_equals_host_blob(name, elem, x):
    hd, hb = lwc.lwc_encode_dfloat11_elements(x, elem)
    t = torch.from_numpy(x.view(np.int32) if elem == 1 else x.view(np.int16)).to("cuda")
    if elem == 2:
        t = t.view(torch.float16)
    elif elem == 1:
        t = t.view(torch.float32)
    dd, db = encode_on_device(t, "dfloat11")
    assert dd.as_dict() == hd.as_dict()
    assert np.array_equal(host_bytes(db), hb)
    assert np.array_equal(odf.decode_elements(hb), x)
