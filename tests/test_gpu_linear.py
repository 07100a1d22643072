"""Decode fused into the linear layer (lwc_linear_dfloat11 / lwc_linear_codebook)
through the C ABI, against the oracle's float64 y = x W^T (oracle/linear.py)
computed from the same synthetic weights and activations.

Tolerance: the library states, per codec, the height h of every output's
FP32 summation tree; products of two BF16 values are exact in FP32, so
|y - exact| <= gamma_h * sum |W x| (oracle.linear.float32_tree_bound). Beside
that bound, one-hot activation rows make every output a single product, so a
sweep over all columns checks every decoded weight bit for bit through the
fused path. Shapes cover rows of 1, ragged column counts (not multiples of
16, 32 or 1024), several tiles and blocks per row, M = 1..8, single-value
tensors, batched calls, and full Llama-3-8B layer shapes (sampled rows)."""
import math

import numpy as np
import pytest
import torch

import synth
from decode_dfloat11_b200 import build as lwc_build
from decode_dfloat11_b200 import lwc
from decode_dfloat11_b200.layers import encode_on_device
from oracle import linear as OL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    lwc_build.build()
    return lwc.load()


def height(codec: str, cols: int, desc) -> int:
    """The summation-tree height the library documents for one output."""
    if codec == "codebook":
        return math.ceil(cols / 32) + 5 if desc.k == 0 else math.ceil(cols / 1024) + 37
    if cols % 16:
        return cols
    return math.ceil(cols / 512) + math.ceil(cols / 32) + 32


def encode(w_u16: np.ndarray, codec: str, **params):
    # "dfloat11_nocounts": a DFloat11 blob without stored chunk counts, which
    # the two-pass fused kernel takes (blobs with counts take the counted one)
    if codec == "dfloat11_nocounts":
        d, b = lwc.lwc_encode_dfloat11(w_u16, chunk_counts=False, **params)
        assert not d.flags & 2
    elif codec == "dfloat11":
        d, b = lwc.lwc_encode_dfloat11(w_u16, **params)
    else:
        d, b = lwc.lwc_encode_codebook(w_u16, **params)
    return d, torch.from_numpy(b).to("cuda")


def run_linear(codec, desc, blob, cols, x, M):
    rows = desc.n // cols
    y = torch.full((M, rows), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fn = lwc.lwc_linear_codebook if codec == "codebook" else lwc.lwc_linear_dfloat11
    fn(desc, blob, cols, x, M, y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return y.cpu().numpy().astype(np.float64)


def check(y, w_u16_rows, x, cols, codec, desc):
    want, mag = OL.linear(w_u16_rows, synth.as_u16(x).reshape(x.shape[0], cols))
    tol = OL.float32_tree_bound(mag, height(codec, cols, desc))
    err = np.abs(y - want)
    assert np.all(err <= tol), (float((err - tol).max()), np.unravel_index(np.argmax(err - tol), err.shape))


SHAPES = [(1, 16), (1, 1), (7, 33), (5, 100), (200, 8), (33, 48), (64, 1024), (17, 1040), (9, 2048 + 48),
          (300, 4096), (3, 14336), (2, 4099)]


@pytest.mark.parametrize("codec", ["dfloat11", "dfloat11_nocounts", "codebook"])
@pytest.mark.parametrize("rows,cols", SHAPES)
@pytest.mark.parametrize("M", [1, 3, 8])
def test_linear_matches_oracle(codec, rows, cols, M):
    w = synth.as_u16(synth.normal_bf16((rows * cols,), seed=rows * 7 + cols, sigma=0.02, outlier_frac=1e-3))
    d, blob = encode(w, codec)
    x = synth.activations_bf16(M, cols, seed=cols + M, device="cuda")
    y = run_linear(codec, d, blob, cols, x, M)
    check(y, w.reshape(rows, cols), x, cols, codec, d)


@pytest.mark.parametrize("codec", ["dfloat11", "dfloat11_nocounts", "codebook"])
@pytest.mark.parametrize("rows,cols", [(40, 48), (9, 100), (3, 1040), (70, 16)])
def test_one_hot_sweep_checks_every_weight_exactly(codec, rows, cols):
    # x row m is one at column c_m: y[m, r] = W[r, c_m] exactly, whatever the order of the sums
    w = synth.as_u16(synth.normal_bf16((rows * cols,), seed=cols, sigma=0.02, outlier_frac=1e-2))
    d, blob = encode(w, codec)
    W = OL.bf16_values(w.reshape(rows, cols))
    for c0 in range(0, cols, 8):
        M = min(8, cols - c0)
        x = torch.zeros((M, cols), dtype=torch.bfloat16, device="cuda")
        for m in range(M):
            x[m, c0 + m] = 1.0
        y = run_linear(codec, d, blob, cols, x, M)
        assert np.array_equal(y, W[:, c0:c0 + M].T), c0


@pytest.mark.parametrize("codec", ["dfloat11", "codebook"])
def test_df11_parameters_and_long_codes(codec):
    rows, cols = 129, 784
    fib = [1, 1]
    while len(fib) < 24:
        fib.append(fib[-1] + fib[-2])
    w = np.repeat((np.arange(24, dtype=np.uint16) + 100) << 7 | 0x0025, fib)[: rows * cols]
    w = np.resize(w, rows * cols)
    w = np.random.default_rng(0).permutation(w).astype(np.uint16)
    x = synth.activations_bf16(4, cols, seed=5, device="cuda")
    params = [{}] if codec == "codebook" else [dict(chunk_bytes=8), dict(chunk_bytes=36, max_len=16),
                                                dict(chunk_bytes=100), dict(chunk_bytes=1024)]
    for p in params:
        d, blob = encode(w, codec, **p)
        y = run_linear(codec, d, blob, cols, x, 4)
        check(y, w.reshape(rows, cols), x, cols, codec, d)


@pytest.mark.parametrize("codec", ["dfloat11", "codebook"])
def test_single_value_and_single_exponent_tensors(codec):
    rows, cols = 50, 96
    const = np.full(rows * cols, 0x3C25, np.uint16)                  # one value (U = 1)
    single_exp = ((np.arange(rows * cols) * 37) & 0x807F | 0x3C00).astype(np.uint16)   # one exponent
    x = synth.activations_bf16(2, cols, seed=9, device="cuda")
    for w in (const, single_exp):
        d, blob = encode(w, codec)
        y = run_linear(codec, d, blob, cols, x, 2)
        check(y, w.reshape(rows, cols), x, cols, codec, d)


@pytest.mark.parametrize("L", [1, 4, 7])
def test_fixed_length_codes(L):
    """Flat exponent histograms over 2^L values: every code word has length L,
    which the counted kernel reads as back-to-back L-bit fields; one-hot rows
    check every weight of a few columns exactly."""
    rows, cols = 37, 1040
    w = synth.as_u16(synth.equal_exponents(rows * cols, L, seed=70 + L))
    d, blob = encode(w, "dfloat11", chunk_bytes=20)
    assert d.flags & 2
    x = synth.activations_bf16(5, cols, seed=L, device="cuda")
    check(run_linear("dfloat11", d, blob, cols, x, 5), w.reshape(rows, cols), x, cols, "dfloat11", d)
    W = OL.bf16_values(w.reshape(rows, cols))
    cs = [0, 1, 511, 1032, 1039]
    x = torch.zeros((len(cs), cols), dtype=torch.bfloat16, device="cuda")
    for m, c in enumerate(cs):
        x[m, c] = 1.0
    assert np.array_equal(run_linear("dfloat11", d, blob, cols, x, len(cs)), W[:, cs].T)


def moderate(w: np.ndarray) -> np.ndarray:
    """Map exponent fields into [49, 205] (values 2^-78 .. 2^79): products with
    activations and their sums stay inside FP32's normal range, where the
    products are exact."""
    e = (w.astype(np.int64) >> 7) & 0xFF
    return ((w & 0x807F) | ((49 + e % 157) << 7)).astype(np.uint16)


@pytest.mark.parametrize("codec", ["dfloat11", "codebook"])
def test_index_widths_and_batched_call(codec):
    # U = 3 .. 40192 distinct patterns (index widths 2 .. 16) plus an empty tensor, in one call
    shapes = [(64, 256, 3), (31, 4096, 300), (8, 1536, 5000), (157, 256, None), (0, 16, 10), (17, 1024, 257)]
    descs, blobs, cols, xs, ys, ws = [], [], [], [], [], []
    for j, (rows, c, U) in enumerate(shapes):
        n = rows * c
        if U is None:   # every pattern with an exponent field in [49, 205], once
            e = np.arange(49, 206, dtype=np.uint16)
            allp = ((e[:, None] << 7) | np.arange(128, dtype=np.uint16)[None, :]).reshape(-1)
            w = np.random.default_rng(j).permutation(np.concatenate([allp, allp | 0x8000]))[:n]
        else:
            w = moderate(synth.as_u16(synth.codebook_stress(U, n, seed=j))) if n else np.zeros(0, np.uint16)
        d, b = encode(w, codec)
        if U is None and codec == "codebook":
            assert d.k == 16
        descs.append(d)
        blobs.append(b)
        cols.append(c)
        xs.append(synth.activations_bf16(3, c, seed=40 + j, device="cuda"))
        ys.append(torch.full((3, rows), float("nan"), dtype=torch.float32, device="cuda"))
        ws.append(w)
    batch = lwc.LinearBatch(descs, blobs, cols, xs, ys, 3)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    (lwc.lwc_linear_dfloat11_batched if codec == "dfloat11" else lwc.lwc_linear_codebook_batched)(batch, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for (rows, c, _), d, x, y, w in zip(shapes, descs, xs, ys, ws):
        if rows:
            check(y.cpu().numpy().astype(np.float64), w.reshape(rows, c), x, c, codec, d)


@pytest.mark.parametrize("codec", ["dfloat11", "codebook"])
@pytest.mark.parametrize("which", ["q", "k", "gate", "down"])
@pytest.mark.parametrize("M", [1, 4])
def test_llama3_8b_layer_shapes_sampled_rows(codec, which, M):
    spec = [s for s in synth.LLAMA3_8B_LAYER if s[0] == which]
    (_, t), = synth.llama_layer_tensors(5, spec, (0.01, 0.04), 0, device="cuda")
    rows, cols = t.shape
    d, blob = encode_on_device(t, codec)
    x = synth.activations_bf16(M, cols, seed=77 + M, device="cuda")
    y = run_linear(codec, d, blob, cols, x, M)
    pick = np.unique(np.concatenate([[0, 1, rows - 2, rows - 1],
                                     np.random.default_rng(rows + M).integers(0, rows, 60)]))
    w_rows = synth.as_u16(t[torch.from_numpy(pick).to("cuda")])
    check(y[:, pick], w_rows.reshape(len(pick), cols), x, cols, codec, d)


def test_linear_argument_errors():
    w = synth.as_u16(synth.normal_bf16((64 * 48,), seed=1, sigma=0.02))
    x = synth.activations_bf16(2, 48, seed=2, device="cuda")
    y = torch.empty((2, 64), dtype=torch.float32, device="cuda")
    for codec in ("dfloat11", "codebook"):
        d, blob = encode(w, codec)
        fn = lwc.lwc_linear_codebook if codec == "codebook" else lwc.lwc_linear_dfloat11
        for M in (0, 9):
            with pytest.raises(lwc.LwcError) as e:
                fn(d, blob, 48, x, M, y)
            assert e.value.status == 1
        for cols in (0, 47, 1 << 31):
            with pytest.raises(lwc.LwcError) as e:
                fn(d, blob, cols, x, 2, y)
            assert e.value.status == 1
        with pytest.raises(lwc.LwcError) as e:
            fn(d, blob, 48, x.view(-1)[1:].data_ptr(), 2, y)   # misaligned activations
        assert e.value.status == 2
    # DFloat11 blobs the fused layer does not take: larger blocks, FP32 elements
    d, blob = encode(w, "dfloat11", threads_per_block=256)
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_linear_dfloat11(d, blob, 48, x, 2, y)
    assert e.value.status == 4
    x32 = np.random.default_rng(3).integers(0, 1 << 30, 64 * 48, dtype=np.uint64).astype(np.uint32)
    d32, b32 = lwc.lwc_encode_dfloat11_elements(x32, lwc.LWC_ELEM_FP32)
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_linear_dfloat11(d32, torch.from_numpy(b32).to("cuda"), 48, x, 2, y)
    assert e.value.status == 4


@pytest.mark.parametrize("codec", ["dfloat11", "codebook"])
def test_resident_model_linear(codec):
    from decode_dfloat11_b200.layers import ResidentModel, fused_linear
    shapes = [(96, 256), (40, 1040), (17, 48)]
    layers = [[synth.normal_bf16(s, 700 + 10 * L + j, sigma=0.02, outlier_frac=1e-3, device="cuda")
               for j, s in enumerate(shapes)] for L in range(2)]
    m = ResidentModel(codec, "cuda")
    for L, ts in enumerate(layers):
        m.add_layer_from_device(f"layer{L}", ts)
    m.finalize()
    for L, ts in enumerate(layers):
        for j, t in enumerate(ts):
            rows, cols = t.shape
            x = synth.activations_bf16(2, cols, seed=50 + j, device="cuda")
            y = m.linear(L, j, x)
            torch.cuda.synchronize()
            check(y.cpu().numpy().astype(np.float64), synth.as_u16(t).reshape(rows, cols), x, cols, codec,
                  m.layers[L]["descs"][j])
    # argument checks of the torch-level helper
    d, b = m.layers[0]["descs"][0], m.layers[0]["blobs"][0]
    with pytest.raises(ValueError):
        fused_linear(d, b, (96, 256), torch.zeros((2, 255), dtype=torch.bfloat16, device="cuda"), codec)
    with pytest.raises(ValueError):
        fused_linear(d, b, (96, 256), torch.zeros((2, 256), dtype=torch.float32, device="cuda"), codec)
    with pytest.raises(ValueError):
        fused_linear(d, b, (96, 256), torch.zeros((2, 256), dtype=torch.bfloat16, device="cuda"), codec,
                     out=torch.empty((2, 95), dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("codec", ["dfloat11", "codebook"])
def test_fused_linear_routes(codec):
    """layers.fused_linear picks the fused kernel or decode-then-GEMM; both
    routes give y = x W^T within their bounds (the GEMM's: gamma_cols, its
    summation order being cuBLAS's), and "auto" sends DFloat11 with more than
    DF11_FUSED_MAX_M rows to the decode route."""
    from decode_dfloat11_b200 import layers
    rows, cols = 300, 1040
    w = synth.as_u16(synth.normal_bf16((rows * cols,), seed=31, sigma=0.02, outlier_frac=1e-3))
    d, blob = encode(w, codec)
    for M in (1, 2, 3, 8):
        x = synth.activations_bf16(M, cols, seed=40 + M, device="cuda")
        want, mag = OL.linear(w.reshape(rows, cols), synth.as_u16(x).reshape(M, cols))
        for route in ("auto", "fused", "decode"):
            y = layers.fused_linear(d, blob, (rows, cols), x, codec, route=route)
            torch.cuda.synchronize()
            taken = "decode" if route == "decode" or (route == "auto" and codec == "dfloat11"
                                                      and M > layers.DF11_FUSED_MAX_M) else "fused"
            h = cols if taken == "decode" else height(codec, cols, d)
            err = np.abs(y.cpu().numpy().astype(np.float64) - want)
            assert np.all(err <= OL.float32_tree_bound(mag, h)), (route, M)
    with pytest.raises(ValueError):
        layers.fused_linear(d, blob, (rows, cols), x, codec, route="gemm")
