"""Decode fused into the tensor-core product (lwc_gemm_dfloat11,
lwc_gemm_dfloat11_batched) and the tile order it reads (lwc_tile_order),
through the C ABI, against the oracle (oracle/linear.py):

* the tile order of a device matrix, bit for bit against
  oracle.linear.tile_order;
* y against the oracle's float64 y = x W^T of the same weights and
  activations, within the bound the library states for the tensor cores:
  |y - exact| <= gamma_cols * sum |W x| with u = 2^-23;
* one-hot activation rows, which make every output one exact product, so a
  sweep over the columns checks every decoded weight, bit for bit, through
  the shared-memory tiles and the MMA;
* M from 1 to 256 (ragged M, the MMA's N padded to a multiple of 16), one
  tile, several 128-row units and k-tiles, batched calls with different
  column counts, the device tile order + device encoder path, the
  Llama-3-8B layer in the launch configuration the bench times (sampled
  rows), repeatability, argument errors and blobs the kernel does not take.
"""
import numpy as np
import pytest
import torch

import synth
from decode_dfloat11_b200 import build as lwc_build
from decode_dfloat11_b200 import lwc
from decode_dfloat11_b200.layers import GEMM_CHUNK_BYTES, TiledWeights
from oracle import linear as OL

pytestmark = pytest.mark.gpu

U_TC = 2.0 ** -23   # unit roundoff the library states for the tensor cores' additions


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    lwc_build.build()
    return lwc.load()


def weights(rows, cols, seed, sigma=0.02):
    t = synth.normal_bf16((rows, cols), seed=seed, sigma=sigma, outlier_frac=0.001)
    return synth.as_u16(t).reshape(rows, cols)


def tiled_blob(w_u16, chunk_bytes=GEMM_CHUNK_BYTES):
    d, b = lwc.lwc_encode_dfloat11(OL.tile_order(w_u16), chunk_bytes=chunk_bytes)
    assert d.flags & 2 and d.threads_per_block == 32
    return d, torch.from_numpy(b).to("cuda")


def run_gemm(d, blob, cols, x, M):
    rows = d.n // cols
    y = torch.full((M, rows), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lwc.lwc_gemm_dfloat11(d, blob, cols, x, M, y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return y.cpu().numpy().astype(np.float64)


def check(y, w_u16, x):
    want, mag = OL.linear(w_u16, synth.as_u16(x).reshape(x.shape[0], -1))
    tol = OL.float32_tree_bound(mag, w_u16.shape[1], unit_roundoff=U_TC)
    err = np.abs(y - want)
    assert np.all(err <= tol), (float((err - tol).max()), np.unravel_index(np.argmax(err - tol), err.shape))


@pytest.mark.parametrize("rows,cols", [(128, 64), (256, 192), (384, 4096)])
def test_tile_order_matches_oracle(rows, cols):
    w = weights(rows, cols, seed=rows * 7 + cols)
    src = torch.from_numpy(w.view(np.int16)).to("cuda")
    dst = torch.empty_like(src)
    lwc.lwc_tile_order(src, rows, cols, dst)
    torch.cuda.synchronize()
    assert np.array_equal(dst.cpu().numpy().view(np.uint16).reshape(-1), OL.tile_order(w))


@pytest.mark.parametrize("chunk", [GEMM_CHUNK_BYTES, 36, 8])
@pytest.mark.parametrize("rows,cols", [(128, 64), (128, 128), (256, 320), (384, 1024)])
@pytest.mark.parametrize("M", [1, 7, 16, 33, 64, 128, 200, 256])
def test_gemm_matches_oracle(rows, cols, M, chunk):
    """16-byte chunks (TiledWeights' default), the encoder's default 36 and
    small 8-byte chunks (blocks of a few hundred weights)."""
    w = weights(rows, cols, seed=rows + cols)
    d, blob = tiled_blob(w, chunk)
    x = synth.activations_bf16(M, cols, seed=M + cols, device="cuda")
    check(run_gemm(d, blob, cols, x, M), w, x)


def test_one_hot_sweep_checks_every_weight_exactly():
    rows, cols, M = 256, 320, 64
    w = weights(rows, cols, seed=5)
    d, blob = tiled_blob(w)
    wv = OL.bf16_values(w)
    for c0 in range(0, cols, M):
        x = torch.zeros((M, cols), dtype=torch.bfloat16, device="cuda")
        x[torch.arange(M), c0 + torch.arange(M)] = 1.0
        y = run_gemm(d, blob, cols, x, M)
        assert np.array_equal(y, wv[:, c0:c0 + M].T)


def test_batched_matrices_with_different_cols():
    M = 40
    shapes = [(256, 256), (128, 256), (256, 768), (384, 64)]
    ws = [weights(r, c, seed=100 + i) for i, (r, c) in enumerate(shapes)]
    enc = [tiled_blob(w) for w in ws]
    xs = [synth.activations_bf16(M, c, seed=200 + i, device="cuda") for i, (_, c) in enumerate(shapes)]
    ys = [torch.full((M, r), float("nan"), dtype=torch.float32, device="cuda") for r, _ in shapes]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    batch = lwc.LinearBatch([d for d, _ in enc], [b for _, b in enc], [c for _, c in shapes], xs, ys, M)
    lwc.lwc_gemm_dfloat11_batched(batch, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for w, x, y in zip(ws, xs, ys):
        check(y.cpu().numpy().astype(np.float64), w, x)


def test_device_tile_order_and_encoder_path():
    """TiledWeights: tile order and compression on the GPU, then the product."""
    rows, cols, M = 384, 512, 96
    w = weights(rows, cols, seed=77)
    tw = TiledWeights(torch.device("cuda"))
    i = tw.add(torch.from_numpy(w.view(np.int16)).to("cuda").view(torch.bfloat16))
    d_host, _ = lwc.lwc_encode_dfloat11(OL.tile_order(w), chunk_bytes=GEMM_CHUNK_BYTES)
    assert tw.descs[i].total_bytes == d_host.total_bytes
    x = synth.activations_bf16(M, cols, seed=78, device="cuda")
    y = tw.gemm(i, x)
    torch.cuda.synchronize()
    check(y.cpu().numpy().astype(np.float64), w, x)


def test_results_repeat_bit_for_bit():
    rows, cols, M = 256, 1024, 128
    w = weights(rows, cols, seed=9)
    d, blob = tiled_blob(w)
    x = synth.activations_bf16(M, cols, seed=10, device="cuda")
    a = run_gemm(d, blob, cols, x, M)
    b = run_gemm(d, blob, cols, x, M)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("M", [16, 128])
def test_llama3_8b_layer_sampled_rows(M):
    """The seven matrices of a Llama-3-8B layer in one batched call (the
    launch the bench times), rows sampled against the oracle."""
    tensors = list(synth.llama_layer_tensors(0, device="cuda"))
    tw = TiledWeights(torch.device("cuda"))
    idx = [tw.add(t) for _, t in tensors]
    xs = [synth.activations_bf16(M, tw.shapes[i][1], seed=300 + i, device="cuda") for i in idx]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ys = tw.gemm_batched(idx, xs, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rng = np.random.default_rng(1)
    for i, (_, t) in zip(idx, tensors):
        rows, cols = tw.shapes[i]
        pick = np.sort(rng.choice(rows, 48, replace=False))
        w_rows = synth.as_u16(t[torch.from_numpy(pick).to("cuda")]).reshape(len(pick), cols)
        want, mag = OL.linear(w_rows, synth.as_u16(xs[i]).reshape(M, cols))
        got = ys[i].cpu().numpy().astype(np.float64)[:, pick]
        assert np.all(np.abs(got - want) <= OL.float32_tree_bound(mag, cols, unit_roundoff=U_TC))


def test_gemm_argument_errors():
    w = weights(256, 128, seed=3)
    d, blob = tiled_blob(w)
    x = synth.activations_bf16(4, 128, seed=4, device="cuda")
    y = torch.empty((300, 256), dtype=torch.float32, device="cuda")
    for M in (0, 257):
        with pytest.raises(lwc.LwcError) as e:
            lwc.lwc_gemm_dfloat11(d, blob, 128, x, M, y)
        assert e.value.status == lwc.LWC_ERR_INVALID_ARG
    for cols in (96, 100, 256 * 128):   # not a multiple of 64; does not divide n; rows not a multiple of 128
        with pytest.raises(lwc.LwcError) as e:
            lwc.lwc_gemm_dfloat11(d, blob, cols, x, 4, y)
        assert e.value.status == lwc.LWC_ERR_INVALID_ARG
    # blobs the kernel does not take: no stored counts, 64-chunk blocks, one exponent value
    tiled = OL.tile_order(w)
    for kw in ({"chunk_counts": False}, {"threads_per_block": 64}):
        d2, b2 = lwc.lwc_encode_dfloat11(tiled, **kw)
        with pytest.raises(lwc.LwcError) as e:
            lwc.lwc_gemm_dfloat11(d2, torch.from_numpy(b2).to("cuda"), 128, x, 4, y)
        assert e.value.status == lwc.LWC_ERR_UNSUPPORTED
    one = np.full(256 * 128, 0x3F80, np.uint16)
    d3, b3 = lwc.lwc_encode_dfloat11(one)
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_gemm_dfloat11(d3, torch.from_numpy(b3).to("cuda"), 128, x, 4, y)
    assert e.value.status == lwc.LWC_ERR_UNSUPPORTED
    # misaligned activations
    xb = torch.empty(4 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_gemm_dfloat11(d, blob, 128, xb[1:1 + 4 * 128], 4, y)
    assert e.value.status == lwc.LWC_ERR_MISALIGNED


def test_tile_order_argument_errors():
    src = torch.zeros(256 * 128, dtype=torch.int16, device="cuda")
    dst = torch.empty_like(src)
    for rows, cols in ((100, 128), (256, 96)):
        with pytest.raises(lwc.LwcError) as e:
            lwc.lwc_tile_order(src, rows, cols, dst)
        assert e.value.status == lwc.LWC_ERR_INVALID_ARG
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_tile_order(src, 256, 128, src)
    assert e.value.status == lwc.LWC_ERR_INVALID_ARG


def test_damaged_blobs_are_reported_and_contained():
    """Damaged tile-order blobs (count bytes, block offsets out of range or
    out of order, every lookup entry invalid, stream bit flips) end the
    product with a device status, within the bounded waits, with nothing
    written outside y; the next call on a sound blob is exact."""
    import time
    rows, cols, M = 384, 1024, 16
    w = weights(rows, cols, seed=21)
    d, b = lwc.lwc_encode_dfloat11(OL.tile_order(w), chunk_bytes=GEMM_CHUNK_BYTES)
    assert d.n_blocks > 8
    rng = np.random.default_rng(3)
    cases = {}
    x = b.copy()
    x[d.off_counts + 32 * 5 + 7] += np.uint8(1)                 # one chunk's code count
    cases["count"] = (x, lwc.LWC_DEVICE_BAD_COUNT)
    x = b.copy()
    x[d.off_blkoff + 8 * 4: d.off_blkoff + 8 * 5] = np.array([2 ** 40], np.uint64).view(np.uint8)
    cases["offset_out_of_range"] = (x, lwc.LWC_DEVICE_BAD_OFFSET | lwc.LWC_DEVICE_BAD_COUNT)
    x = b.copy()
    off = np.frombuffer(x[d.off_blkoff: d.off_blkoff + 8 * (d.n_blocks + 1)].tobytes(), np.uint64).copy()
    off[[2, 6]] = off[[6, 2]]                                   # offsets out of order
    x[d.off_blkoff: d.off_blkoff + 8 * (d.n_blocks + 1)] = off.view(np.uint8)
    cases["offsets_out_of_order"] = (x, lwc.LWC_DEVICE_BAD_OFFSET | lwc.LWC_DEVICE_BAD_COUNT)
    x = b.copy()
    x[d.off_lut: d.off_lut + 512 * d.n_tables] = 0xFF             # every lookup entry invalid
    cases["lut"] = (x, lwc.LWC_DEVICE_BAD_CODE | lwc.LWC_DEVICE_BAD_COUNT)
    x = b.copy()
    x[d.off_stream + rng.integers(0, (d.total_bits + 7) // 8, 50)] ^= np.uint8(0x10)
    cases["bit_flips"] = (x, None)
    guard = 4096
    xa = synth.activations_bf16(M, cols, seed=22, device="cuda")
    for name, (blob, expect) in cases.items():
        ybuf = torch.zeros(M * rows + 2 * guard, dtype=torch.float32, device="cuda")
        y = ybuf[guard:guard + M * rows].view(M, rows)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        t0 = time.perf_counter()
        lwc.lwc_gemm_dfloat11(d, torch.from_numpy(blob).to("cuda"), cols, xa, M, y, status)
        torch.cuda.synchronize()
        assert time.perf_counter() - t0 < 30, name
        got = ybuf.cpu().numpy()
        assert np.all(got[:guard] == 0) and np.all(got[guard + M * rows:] == 0), name
        st = int(status.item())
        if expect is not None:
            assert st & expect, (name, st)
    # the context still computes exactly
    x1 = torch.zeros((64, cols), dtype=torch.bfloat16, device="cuda")
    x1[torch.arange(64), torch.arange(64)] = 1.0
    d0, b0 = tiled_blob(w)
    y = run_gemm(d0, b0, cols, x1, 64)
    assert np.array_equal(y, OL.bf16_values(w)[:, :64].T)


# ---- the codebook codec -----------------------------------------------------------

def cb_tiled_blob(w_u16):
    d, b = lwc.lwc_encode_codebook(OL.tile_order(w_u16))
    return d, torch.from_numpy(b).to("cuda")


def run_cb_gemm(d, blob, cols, x, M):
    rows = d.n // cols
    y = torch.full((M, rows), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lwc.lwc_gemm_codebook(d, blob, cols, x, M, y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return y.cpu().numpy().astype(np.float64)


def few_values(rows, cols, U, seed):
    """A matrix drawing from U distinct BF16 values (index width ceil(log2 U))."""
    vals = synth.as_u16(synth.normal_bf16((U * 4,), seed=seed, sigma=0.02))
    vals = np.unique(vals)[:U]
    rng = np.random.default_rng(seed)
    return vals[rng.integers(0, len(vals), rows * cols)].reshape(rows, cols)


@pytest.mark.parametrize("rows,cols", [(128, 64), (256, 320), (384, 1024)])
@pytest.mark.parametrize("M", [1, 16, 33, 128, 256])
def test_codebook_gemm_matches_oracle(rows, cols, M):
    w = weights(rows, cols, seed=rows * 3 + cols)
    d, blob = cb_tiled_blob(w)
    assert d.k >= 1
    x = synth.activations_bf16(M, cols, seed=M + 7, device="cuda")
    check(run_cb_gemm(d, blob, cols, x, M), w, x)


@pytest.mark.parametrize("U,M", [(2, 16), (3, 64), (17, 16), (255, 128), (1000, 40), (40000, 16), (65536, 16)])
def test_codebook_gemm_index_widths(U, M):
    rows, cols = 256, 192
    w = few_values(rows, cols, U, seed=U) if U < 65536 else \
        synth.as_u16(synth.uniform_patterns(rows * cols, seed=5)).reshape(rows, cols)
    w = np.where(np.isfinite(OL.bf16_values(w)) & (np.abs(OL.bf16_values(w)) < 1e30), w, np.uint16(0x3F80))
    d, blob = cb_tiled_blob(w)
    x = synth.activations_bf16(M, cols, seed=U, device="cuda")
    check(run_cb_gemm(d, blob, cols, x, M), w, x)


def test_codebook_one_hot_sweep_checks_every_weight_exactly():
    rows, cols, M = 256, 320, 64
    w = weights(rows, cols, seed=15)
    d, blob = cb_tiled_blob(w)
    wv = OL.bf16_values(w)
    for c0 in range(0, cols, M):
        x = torch.zeros((M, cols), dtype=torch.bfloat16, device="cuda")
        x[torch.arange(M), c0 + torch.arange(M)] = 1.0
        assert np.array_equal(run_cb_gemm(d, blob, cols, x, M), wv[:, c0:c0 + M].T)


@pytest.mark.parametrize("M", [16, 128])
def test_codebook_llama3_8b_layer_sampled_rows(M):
    tensors = list(synth.llama_layer_tensors(1, device="cuda"))
    tw = TiledWeights(torch.device("cuda"), codec="codebook")
    idx = [tw.add(t) for _, t in tensors]
    ks = {tw.descs[i].k for i in idx}
    xs = [synth.activations_bf16(M, tw.shapes[i][1], seed=400 + i, device="cuda") for i in idx]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if len(ks) > 1:   # one launch takes one index width: group by k
        ys = [None] * len(idx)
        for k in ks:
            sel = [i for i in idx if tw.descs[i].k == k]
            for i, y in zip(sel, tw.gemm_batched(sel, [xs[i] for i in sel], status=status)):
                ys[i] = y
    else:
        ys = tw.gemm_batched(idx, xs, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rng = np.random.default_rng(2)
    for i, (_, t) in zip(idx, tensors):
        rows, cols = tw.shapes[i]
        pick = np.sort(rng.choice(rows, 48, replace=False))
        w_rows = synth.as_u16(t[torch.from_numpy(pick).to("cuda")]).reshape(len(pick), cols)
        want, mag = OL.linear(w_rows, synth.as_u16(xs[i]).reshape(M, cols))
        got = ys[i].cpu().numpy().astype(np.float64)[:, pick]
        assert np.all(np.abs(got - want) <= OL.float32_tree_bound(mag, cols, unit_roundoff=U_TC))


def test_codebook_gemm_argument_errors():
    w = weights(256, 128, seed=31)
    d, blob = cb_tiled_blob(w)
    x = synth.activations_bf16(4, 128, seed=32, device="cuda")
    y = torch.empty((4, 256), dtype=torch.float32, device="cuda")
    d1, b1 = lwc.lwc_encode_codebook(np.full(256 * 128, 0x3F80, np.uint16))   # one value: k = 0
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_gemm_codebook(d1, torch.from_numpy(b1).to("cuda"), 128, x, 4, y)
    assert e.value.status == lwc.LWC_ERR_UNSUPPORTED
    w2 = few_values(256, 128, 5, seed=33)
    d2, b2 = cb_tiled_blob(w2)
    assert d2.k != d.k
    yb = [torch.empty((4, 256), dtype=torch.float32, device="cuda") for _ in range(2)]
    batch = lwc.LinearBatch([d, d2], [blob, b2], [128, 128], [x, x], yb, 4)
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_gemm_codebook_batched(batch)
    assert e.value.status == lwc.LWC_ERR_UNSUPPORTED
    dd, bd = tiled_blob(w)   # a DFloat11 blob is not a codebook blob
    with pytest.raises(lwc.LwcError):
        lwc.lwc_gemm_codebook(dd, bd, 128, x, 4, y)
