"""Model-scale decodes: compressed weights resident in HBM, decoded layer by
layer (one batched launch per layer) into reusable BF16 ping-pong buffers.

Full Llama-3-8B shapes (32 layers + embedding + LM head, 8.03 B weights) with
both codecs resident at once, and Llama-3-70B shapes (three layers resident
with the embedding and LM head; and all 82 units decoded one at a time). Every decoded
layer is compared, on the device, with the same seeded tensors generated
again; the oracle decodes sampled blobs on the host for an independent check."""
import numpy as np
import pytest
import torch

import synth
from decode_dfloat11_b200 import build as lwc_build
from decode_dfloat11_b200 import lwc
from decode_dfloat11_b200.layers import ResidentModel, encode_many
from oracle import codebook as ocb
from oracle import df11 as odf

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    lwc_build.build()
    return lwc.load()


def model_units(which: str, layers):
    """(name, generator) per unit; a generator yields the unit's tensors on the GPU."""
    if which == "8b":
        hidden, shapes, sig, off = synth.LLAMA3_8B_HIDDEN, synth.LLAMA3_8B_LAYER, (0.01, 0.04), 0
    else:
        hidden, shapes, sig, off = synth.LLAMA3_70B_HIDDEN, synth.LLAMA3_70B_LAYER, (0.005, 0.03), \
            synth.SEED_70B_OFFSET
    units = [("embed", lambda: [synth.llama_embedding("embed", hidden, sig, off, device="cuda")])]
    for L in layers:
        units.append((f"layer{L}", lambda L=L: [t for _, t in synth.llama_layer_tensors(
            L, shapes, sig, off, device="cuda")]))
    units.append(("lm_head", lambda: [synth.llama_embedding("lm_head", hidden, sig, off, device="cuda")]))
    return units


def build(units, codecs):
    models = {c: ResidentModel(c, "cuda") for c in codecs}
    for name, gen in units:
        tensors = gen()
        host = [synth.as_u16(t) for t in tensors]
        shapes = [t.shape for t in tensors]
        del tensors
        for c, m in models.items():
            m.add_layer(name, encode_many(host, c), shapes)
    for m in models.values():
        m.finalize()
    return models


def check_all(units, models, oracle_units=()):
    stream = torch.cuda.current_stream()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for i, (name, gen) in enumerate(units):
        expect = gen()
        for c, m in models.items():
            slot = i % 2
            m.decode(i, slot, stream, status)
            torch.cuda.synchronize()
            for v, t in zip(m.views(i, slot), expect):
                assert torch.equal(v.view(torch.int16), t.view(torch.int16)), (c, name)
            if name in oracle_units:
                got = m.views(i, slot)[0].reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16)
                blob = m.layers[i]["blobs"][0].cpu().numpy()
                ref = odf.decode(blob) if c == "dfloat11" else ocb.decode(blob)
                assert np.array_equal(got, ref), (c, name)
        del expect
    assert int(status.item()) == 0


def test_llama3_8b_model_both_codecs_resident():
    units = model_units("8b", range(synth.LLAMA3_8B_LAYERS))
    models = build(units, ("dfloat11", "codebook"))
    df, cb = models["dfloat11"], models["codebook"]
    assert df.weights == cb.weights == 8_029_995_008
    assert 10.0 < 8 * df.compressed_bytes / df.weights < 11.5
    assert 12.5 < 8 * cb.compressed_bytes / cb.weights < 14.5
    check_all(units, models, oracle_units=("layer0", "lm_head"))


def test_llama3_70b_layers_full_shapes():
    units = model_units("70b", (0, 41, 79))
    models = build(units, ("dfloat11",))
    df = models["dfloat11"]
    assert 10.0 < 8 * df.compressed_bytes / df.weights < 11.5
    check_all(units, models, oracle_units=("layer41",))


def test_llama3_70b_every_unit_decodes_exactly():
    """All 82 units of the Llama-3-70B-shaped model (embedding, the 80
    decoder layers, LM head: 70.55 B weights), each generated on the GPU,
    compressed there (device encoder, the blob format the bench keeps
    resident) and decoded in one batched launch, compared bit for bit with
    the regenerated tensors. One unit at a time, so the test holds a few GB."""
    from decode_dfloat11_b200.layers import encode_on_device
    units = model_units("70b", range(synth.LLAMA3_70B_LAYERS))
    stream = torch.cuda.current_stream()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    biggest = synth.VOCAB * synth.LLAMA3_70B_HIDDEN   # the embedding and LM head
    work = torch.empty(lwc.lwc_encode_device_workspace_bytes(biggest), dtype=torch.uint8, device="cuda")
    total = 0
    for name, gen in units:
        tensors = gen()
        enc = [encode_on_device(t, "dfloat11", workspace=work) for t in tensors]
        outs = [torch.empty(t.numel(), dtype=torch.int16, device="cuda") for t in tensors]
        lwc.lwc_decode_dfloat11_batched(lwc.Batch([d for d, _ in enc], [b for _, b in enc], outs),
                                        d_status=status, stream=stream)
        assert all(d.flags & 2 for d, _ in enc), name       # stored chunk counts: the counted decoder
        for o, t in zip(outs, tensors):
            assert torch.equal(o, t.reshape(-1).view(torch.int16)), name
        total += sum(t.numel() for t in tensors)
        del tensors, enc, outs
    assert total == 70_552_387_584
    assert int(status.item()) == 0


def test_pipelined_decode_overlaps_and_never_clobbers():
    """Layer L+1 decodes on a side stream while layer L is consumed; the
    consumer copies every weight it sees and runs a GEMM on it, so a buffer
    overwritten too early would show up as a mismatch."""
    shapes = [(3072, 1024), (1024, 3072), (2048, 2048)]
    units = []
    for L in range(6):
        units.append((f"layer{L}", lambda L=L: [synth.normal_bf16(s, 7000 + 10 * L + j, sigma=0.02,
                                                                outlier_frac=1e-3, device="cuda")
                                                for j, s in enumerate(shapes)]))
    model = build(units, ("dfloat11",))["dfloat11"]
    compute = torch.cuda.Stream()
    x = torch.randn(64, 1024, device="cuda", dtype=torch.bfloat16)
    compute.wait_stream(torch.cuda.current_stream())
    copies, outs = [], []
    with torch.cuda.stream(compute):
        for i, views in model.pipelined(compute):
            copies.append([v.clone() for v in views])
            outs.append(torch.relu(x @ views[1]))   # some real work on the decoded (1024 x 3072) matrix
    torch.cuda.synchronize()
    for (name, gen), got in zip(units, copies):
        for g, t in zip(got, gen()):
            assert torch.equal(g.view(torch.int16), t.view(torch.int16)), name
    assert all(o.shape == (64, 3072) for o in outs)


def test_layer_decodes_replay_from_a_cuda_graph():
    """The decoders only enqueue kernels (no allocation, no synchronisation),
    so a whole model's layer-by-layer decode can be captured once into a CUDA
    graph and replayed; the first (uncaptured) call does the per-device setup."""
    shapes = [(3072, 1024), (1024, 3072), (2048, 2048)]
    units = [(f"layer{L}", lambda L=L: [synth.normal_bf16(s, 8000 + 10 * L + j, sigma=0.02, outlier_frac=1e-3,
                                                          device="cuda") for j, s in enumerate(shapes)])
             for L in range(4)]
    models = build(units, ("dfloat11", "codebook"))
    stream = torch.cuda.Stream()
    sinks = {c: [torch.empty(sum(int(np.prod(s)) for s in shapes), dtype=torch.bfloat16, device="cuda")
                 for _ in units] for c in models}
    with torch.cuda.stream(stream):
        for c, m in models.items():          # setup outside the capture
            m.decode(0, 0, stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for c, m in models.items():
            for i in range(len(units)):
                m.decode(i, i % 2, stream)
                off = 0
                for v in m.views(i, i % 2):   # copy each decoded layer out of the ping-pong buffer
                    sinks[c][i][off:off + v.numel()].copy_(v.reshape(-1))
                    off += v.numel()
    for _ in range(2):
        for c in sinks:
            for t in sinks[c]:
                t.zero_()
        graph.replay()
        torch.cuda.synchronize()
        for c in models:
            for (name, gen), got in zip(units, sinks[c]):
                want = torch.cat([t.reshape(-1) for t in gen()])
                assert torch.equal(got.view(torch.int16), want.view(torch.int16)), (c, name)


@pytest.mark.parametrize("codec", ["dfloat11", "codebook"])
def test_host_pipeline_round_trip(codec):
    """Host blobs -> GPU decode -> host output with overlapped transfers
    (layers.HostPipeline), run twice on the same buffers."""
    from decode_dfloat11_b200.layers import HostPipeline
    ws = [synth.as_u16(synth.normal_bf16((n,), seed=9100 + n, sigma=0.02, outlier_frac=1e-3))
          for n in (1_000_003, 17, 4_194_304, 65_537)]
    enc = encode_many(ws, codec)
    pipe = HostPipeline([d for d, _ in enc], [b for _, b in enc], codec, "cuda")
    stream = torch.cuda.current_stream()
    for _ in range(2):
        pipe.host_out.zero_()
        pipe.run(stream)
        stream.synchronize()
        got = pipe.host_out.view(torch.int16).numpy().view(np.uint16)
        for w, off in zip(ws, pipe.offsets):
            assert np.array_equal(got[off:off + w.size], w)
    assert pipe.h2d_bytes == sum(b.size for _, b in enc) and pipe.d2h_bytes == 2 * sum(w.size for w in ws)
