"""Compressed model weights resident in GPU memory, decoded layer by layer.

This follows the DFloat11 page ("Koniec z kompromisami! DFloat11 ratuje
dokładność modeli AI ...", section "Jak to działa w praktyce? Magia na
poziomie GPU", third pillar): the weights stay compressed in HBM and all the
matrices of one transformer block are decompressed together, in one launch,
right before the block runs. Decoded layers land in a small set of reusable
BF16 buffers (two by default: a ping-pong pair, so layer L+1 can be decoded
while layer L is in use).

Everything here is bookkeeping and argument marshalling around the C ABI
(``lwc_decode_dfloat11_batched`` / ``lwc_decode_codebook_batched``); the
decoding itself runs in liblwc's CUDA kernels.
"""
from __future__ import annotations

import concurrent.futures as cf
import os


from . import lwc

CODECS = ("dfloat11", "codebook")


def encode_many(arrays, codec: str = "dfloat11", workers: int | None = None, **params):
    """Encode host BF16 bit-pattern arrays in parallel host threads (the C
    encoder releases the GIL). Returns [(desc, blob), ...] in input order."""
    if codec not in CODECS:
        raise ValueError(f"unknown codec {codec!r}")
    fn = (lambda a: lwc.lwc_encode_dfloat11(a, **params)) if codec == "dfloat11" else lwc.lwc_encode_codebook
    workers = workers or min(len(arrays), os.cpu_count() or 1) or 1
    with cf.ThreadPoolExecutor(max_workers=workers) as ex:
        return list(ex.map(fn, arrays))


def encode_on_device(tensor, codec: str = "dfloat11", workspace=None, stream=None, **params):
    """Compress a tensor that is already on the GPU into a device blob
    (``lwc_encode_*_device_plan`` + ``lwc_encode_device_write``). BF16 (or any
    16-bit patterns) for both codecs; float32 / float16 tensors with the
    DFloat11 codec use its FP32 / FP16 element types.

    Returns ``(desc, blob)`` with ``blob`` a uint8 CUDA tensor of
    ``desc.total_bytes`` bytes, byte-for-byte what the host encoder would make.
    ``workspace`` (a uint8 CUDA tensor of at least
    ``lwc_encode_device_workspace_bytes(n)`` bytes) may be passed to reuse one
    buffer across tensors; the tensor must not change while this runs."""
    import torch
    if codec not in CODECS:
        raise ValueError(f"unknown codec {codec!r}")
    src = tensor.reshape(-1).contiguous()
    elem = lwc.LWC_ELEM_BF16
    if src.dtype == torch.float32 or src.dtype == torch.int32:
        elem = lwc.LWC_ELEM_FP32
    elif src.dtype == torch.float16:
        elem = lwc.LWC_ELEM_FP16
    elif src.element_size() != 2:
        raise ValueError("expected a 16-bit or 32-bit tensor")
    if elem != lwc.LWC_ELEM_BF16 and codec != "dfloat11":
        raise ValueError("FP32 / FP16 element types are a DFloat11 feature (the codebook takes 16-bit patterns)")
    n = src.numel()
    need = lwc.lwc_encode_device_workspace_bytes(n)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=src.device)
    work_bytes = workspace.numel()
    stream = stream if stream is not None else torch.cuda.current_stream(src.device)
    if codec == "dfloat11":
        desc = lwc.lwc_encode_dfloat11_elements_device_plan(src, n, elem, workspace, work_bytes, stream=stream,
                                                            **params)
    else:
        desc = lwc.lwc_encode_codebook_device_plan(src, n, workspace, work_bytes, stream=stream)
    blob = torch.empty(desc.total_bytes, dtype=torch.uint8, device=src.device)
    desc = lwc.lwc_encode_device_write(src, n, workspace, work_bytes, blob, blob.numel(), stream=stream)
    return desc, blob


# Activation rows from which the DFloat11 decode-fused linear layer is slower
# than decoding the matrix and running the GEMM (Llama-3-8B layer on B200:
# fused 1.43 x faster at M = 1, 0.88 x at M = 4).
DF11_FUSED_MAX_M = 2


def fused_linear(desc, blob, shape, x, codec: str, out=None, stream=None, status=None, route: str = "auto"):
    """y = x W^T with W (``shape`` = (rows, cols), the tensor ``blob``
    decodes to); x: M x cols BF16 on the GPU, M <= 8. Returns ``out`` (M x
    rows FP32, allocated if None).

    route "fused": the decode-fused kernel (W decoded in registers, never
    written); "decode": decode W into a BF16 buffer, then a BF16 x BF16 ->
    FP32 GEMM (torch.mm; its summation order is cuBLAS's, so the bound is
    gamma_cols); "auto": fused, except DFloat11 with more than
    DF11_FUSED_MAX_M rows, where the fused kernel is the slower of the two."""
    import torch
    if codec not in CODECS:
        raise ValueError(f"unknown codec {codec!r}")
    if route not in ("auto", "fused", "decode"):
        raise ValueError(f"unknown route {route!r}")
    if len(shape) != 2:
        raise ValueError("the weight must be a rows x cols matrix")
    rows, cols = int(shape[0]), int(shape[1])
    if x.dim() != 2 or x.shape[1] != cols or x.dtype != torch.bfloat16:
        raise ValueError(f"x must be M x {cols} BF16")
    x = x.contiguous()
    M = int(x.shape[0])
    if out is None:
        out = torch.empty((M, rows), dtype=torch.float32, device=x.device)
    elif tuple(out.shape) != (M, rows) or out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {M} x {rows} FP32 tensor")
    if route == "auto":
        route = "decode" if codec == "dfloat11" and M > DF11_FUSED_MAX_M else "fused"
    if route == "decode":
        s = stream if stream is not None else torch.cuda.current_stream(x.device)
        w = torch.empty((rows, cols), dtype=torch.bfloat16, device=x.device)
        dec = lwc.lwc_decode_dfloat11_checked if codec == "dfloat11" else lwc.lwc_decode_codebook_checked
        dec(desc, blob, w, status, s)
        with torch.cuda.stream(s):
            out.copy_(torch.mm(x, w.t(), out_dtype=torch.float32))
        return out
    fn = lwc.lwc_linear_dfloat11 if codec == "dfloat11" else lwc.lwc_linear_codebook
    fn(desc, blob, cols, x, M, out, d_status=status, stream=stream)
    return out


# Chunk size of the blobs TiledWeights makes. A 32-chunk block of 20-byte
# chunks holds about 2,000 exponent codes, so the product can run 20 decoder
# warps with about five 8192-weight tiles in flight (36-byte chunks: 12 warps);
# the price is 0.13 bits per weight of chunk gaps and counts. Measured on a
# Llama-3-8B layer (B200), M = 16 / 128 / 256: 20-byte chunks 0.31 / 0.34 /
# 0.42 ms; 24: 0.31 / 0.34 / 0.50; 28: 0.29 / 0.38 / 0.59; 36: 0.32 / 0.41 / 0.67.
GEMM_CHUNK_BYTES = 20


class TiledWeights:
    """Weight matrices held for the tensor-core product (lwc_gemm_dfloat11 /
    lwc_gemm_codebook): each rows x cols BF16 matrix (rows % 128 == 0, cols %
    64 == 0) is put in tile order on the GPU (lwc_tile_order) and compressed
    there by the device encoder of ``codec``. ``gemm`` then computes y = x W^T
    for 1 to 256 activation rows with W decoded straight into the MMA's
    shared-memory operands (the BF16 matrix is never written to device
    memory). A batched call takes matrices of one codec (codebook: one index
    width)."""

    def __init__(self, device, codec: str = "dfloat11"):
        if codec not in CODECS:
            raise ValueError(f"unknown codec {codec!r}")
        self.device = device
        self.codec = codec
        self.descs, self.blobs, self.shapes = [], [], []

    def add(self, w, workspace=None, stream=None, chunk_bytes: int = GEMM_CHUNK_BYTES) -> int:
        """Tile-order and compress one rows x cols BF16 CUDA tensor; returns its index.
        chunk_bytes: DFloat11 chunk size of the blob (see GEMM_CHUNK_BYTES)."""
        import torch
        if w.dim() != 2 or w.element_size() != 2 or not w.is_cuda:
            raise ValueError("expected a rows x cols 16-bit CUDA tensor")
        rows, cols = int(w.shape[0]), int(w.shape[1])
        stream = stream if stream is not None else torch.cuda.current_stream(w.device)
        src = w.contiguous()
        tiled = torch.empty_like(src)
        lwc.lwc_tile_order(src, rows, cols, tiled, stream)
        with torch.cuda.stream(stream):
            params = {"chunk_bytes": chunk_bytes} if self.codec == "dfloat11" else {}
            d, b = encode_on_device(tiled, self.codec, workspace=workspace, stream=stream, **params)
        del tiled
        self.descs.append(d)
        self.blobs.append(b)
        self.shapes.append((rows, cols))
        return len(self.descs) - 1

    @property
    def compressed_bytes(self) -> int:
        return sum(int(d.total_bytes) for d in self.descs)

    def _check_x(self, index: int, x):
        import torch
        rows, cols = self.shapes[index]
        if x.dim() != 2 or x.shape[1] != cols or x.dtype != torch.bfloat16:
            raise ValueError(f"x must be M x {cols} BF16")
        return rows, cols, x.contiguous()

    def gemm(self, index: int, x, out=None, stream=None, status=None):
        """y = x W^T for matrix ``index``; x: M x cols BF16 (M <= 256). Returns
        ``out`` (M x rows FP32, allocated if None)."""
        import torch
        rows, cols, x = self._check_x(index, x)
        M = int(x.shape[0])
        if out is None:
            out = torch.empty((M, rows), dtype=torch.float32, device=x.device)
        fn = lwc.lwc_gemm_dfloat11 if self.codec == "dfloat11" else lwc.lwc_gemm_codebook
        fn(self.descs[index], self.blobs[index], cols, x, M, out, d_status=status, stream=stream)
        return out

    def gemm_batched(self, indices, xs, outs=None, stream=None, status=None):
        """Several matrices (at most 8), one launch; all x share M."""
        import torch
        xs = [self._check_x(i, x)[2] for i, x in zip(indices, xs)]
        M = int(xs[0].shape[0])
        if any(int(x.shape[0]) != M for x in xs):
            raise ValueError("all activations of a batched call share M")
        if outs is None:
            outs = [torch.empty((M, self.shapes[i][0]), dtype=torch.float32, device=xs[0].device) for i in indices]
        batch = lwc.LinearBatch([self.descs[i] for i in indices], [self.blobs[i] for i in indices],
                                [self.shapes[i][1] for i in indices], xs, outs, M)
        fn = lwc.lwc_gemm_dfloat11_batched if self.codec == "dfloat11" else lwc.lwc_gemm_codebook_batched
        fn(batch, d_status=status, stream=stream)
        return outs


class ResidentModel:
    """Compressed layers in device memory plus reusable BF16 output buffers.

    Usage: ``add_layer`` for every layer (uploads its blobs), ``finalize`` to
    allocate the buffers and marshal the launch arguments once, then
    ``decode(layer, slot, stream)`` per layer; ``views(layer, slot)`` gives
    the decoded matrices (BF16 views into buffer ``slot``).
    """

    def __init__(self, codec: str, device, slots: int = 2):
        import torch
        if codec not in CODECS:
            raise ValueError(f"unknown codec {codec!r}")
        if slots < 2:
            # pipelined() decodes layer L + 1 while layer L is still in use:
            # that needs a second buffer
            raise ValueError(f"ResidentModel needs at least 2 output buffers (got slots={slots})")
        self.codec = codec
        self.device = torch.device(device)
        self.slots = slots
        self.layers: list[dict] = []
        self.buffers = []
        self._batches: list[list] = []

    def add_layer(self, name: str, encoded, shapes) -> None:
        """encoded: [(desc, host blob)] of the layer's matrices, shapes their shapes."""
        import torch
        descs = [d for d, _ in encoded]
        blobs = [torch.from_numpy(b).to(self.device) for _, b in encoded]
        self.layers.append(dict(name=name, descs=descs, blobs=blobs, shapes=[tuple(s) for s in shapes],
                                n=[d.n for d in descs]))

    def add_layer_from_device(self, name: str, tensors, workspace=None, **params) -> None:
        """Compress BF16 tensors that are already on this model's GPU (the
        device encoder) and keep only their blobs."""
        import torch
        encoded = []
        for t in tensors:
            need = lwc.lwc_encode_device_workspace_bytes(t.numel())
            if workspace is None or workspace.numel() < need:
                workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
            encoded.append(encode_on_device(t, self.codec, workspace, **params))
        self.layers.append(dict(name=name, descs=[d for d, _ in encoded], blobs=[b for _, b in encoded],
                                shapes=[tuple(t.shape) for t in tensors], n=[d.n for d, _ in encoded]))

    @property
    def compressed_bytes(self) -> int:
        return sum(int(b.numel()) for layer in self.layers for b in layer["blobs"])

    @property
    def weights(self) -> int:
        return sum(sum(layer["n"]) for layer in self.layers)

    def finalize(self) -> None:
        import torch
        biggest = max(sum(layer["n"]) for layer in self.layers)
        # 8 extra elements per matrix keep every view 16-byte aligned
        biggest += 8 * max(len(layer["n"]) for layer in self.layers)
        self.buffers = [torch.empty(biggest, dtype=torch.bfloat16, device=self.device) for _ in range(self.slots)]
        self._batches = []
        for layer in self.layers:
            per_slot = []
            for s in range(self.slots):
                views = self._views(layer, s)
                per_slot.append((lwc.Batch(layer["descs"], layer["blobs"], views), views))
            self._batches.append(per_slot)

    def _views(self, layer, slot):
        out, off = [], 0
        for n, shape in zip(layer["n"], layer["shapes"]):
            out.append(self.buffers[slot][off:off + n].view(shape))
            off += (n + 7) // 8 * 8
        return out

    def views(self, layer: int, slot: int):
        return self._batches[layer][slot][1]

    def decode(self, layer: int, slot: int, stream=None, status=None) -> None:
        batch = self._batches[layer][slot][0]
        if self.codec == "dfloat11":
            lwc.lwc_decode_dfloat11_batched(batch, d_status=status, stream=stream)
        else:
            lwc.lwc_decode_codebook_batched(batch, d_status=status, stream=stream)

    def linear(self, layer: int, index: int, x, out=None, stream=None, status=None, route: str = "auto"):
        """y = x W^T for matrix ``index`` of ``layer``, by default without
        decoding it to memory: the weights are decoded in registers by the
        fused kernel (lwc_linear_dfloat11 / lwc_linear_codebook); see
        fused_linear for ``route``. x: M x cols BF16 on this model's GPU,
        1 <= M <= 8 (token generation); returns (or fills ``out``) the M x rows
        FP32 result."""
        return fused_linear(self.layers[layer]["descs"][index], self.layers[layer]["blobs"][index],
                            self.layers[layer]["shapes"][index], x, self.codec, out=out, stream=stream,
                            status=status, route=route)

    def pipelined(self, compute_stream, decode_stream=None):
        """Iterate over the layers with decoding one layer ahead of use.

        Yields ``(layer, views)``; the views are ready for work enqueued on
        ``compute_stream``, and layer + 1 is already being decoded on
        ``decode_stream`` meanwhile (a side stream if None). Enqueue all work
        that reads the yielded views on ``compute_stream`` before advancing
        the generator: a buffer is reused only after an event recorded on
        ``compute_stream`` at that point says its consumer has finished.
        """
        import torch
        ds = decode_stream or torch.cuda.Stream(self.device)
        ready = [torch.cuda.Event() for _ in range(self.slots)]
        free = [torch.cuda.Event() for _ in range(self.slots)]
        used = [False] * self.slots
        ds.wait_stream(compute_stream)   # inputs written before the call are visible
        self.decode(0, 0, ds)
        ready[0].record(ds)
        for i in range(len(self.layers)):
            slot = i % self.slots
            nxt = i + 1
            if nxt < len(self.layers):
                ns = nxt % self.slots
                if used[ns]:
                    ds.wait_event(free[ns])
                self.decode(nxt, ns, ds)
                ready[ns].record(ds)
            compute_stream.wait_event(ready[slot])
            yield i, self.views(i, slot)
            free[slot].record(compute_stream)
            used[slot] = True


class HostPipeline:
    """Compressed tensors held in (pinned) host memory, decoded through the GPU
    back into host memory, with the transfers overlapped: tensor i's upload,
    tensor i-1's decode and tensor i-2's read-back run on three streams, so
    both PCIe directions are busy at once (smallest tensors first, so the
    read-back starts early).

    ``run()`` enqueues one pass on ``stream`` (and two helper streams) and
    returns; work after it on ``stream`` sees the host output complete once
    the stream is synchronised.
    """

    def __init__(self, descs, host_blobs, codec: str, device, host_out=None):
        import torch
        if codec not in CODECS:
            raise ValueError(f"unknown codec {codec!r}")
        self.codec = codec
        self.device = torch.device(device)
        self.descs = list(descs)
        self.pinned_in = [b if isinstance(b, torch.Tensor) and b.is_pinned() else
                          torch.as_tensor(b).pin_memory() for b in host_blobs]
        self.blobs = [torch.empty(b.numel(), dtype=torch.uint8, device=self.device) for b in self.pinned_in]
        ns = [d.n for d in self.descs]
        self.offsets = []            # element offsets, multiples of 8 (16-byte aligned views)
        off = 0
        for n in ns:
            self.offsets.append(off)
            off += (n + 7) // 8 * 8
        self.out = torch.empty(off, dtype=torch.bfloat16, device=self.device)
        self.host_out = host_out if host_out is not None else torch.empty(off, dtype=torch.bfloat16).pin_memory()
        self.views = [self.out[o:o + n] for o, n in zip(self.offsets, ns)]
        self.order = sorted(range(len(ns)), key=lambda i: ns[i])
        self.s_in = torch.cuda.Stream(self.device)
        self.s_out = torch.cuda.Stream(self.device)

    @property
    def h2d_bytes(self) -> int:
        return sum(int(b.numel()) for b in self.pinned_in)

    @property
    def d2h_bytes(self) -> int:
        return 2 * sum(d.n for d in self.descs)

    def run(self, stream) -> None:
        import torch
        decode = lwc.lwc_decode_dfloat11 if self.codec == "dfloat11" else lwc.lwc_decode_codebook
        self.s_in.wait_stream(stream)        # earlier work on `stream` is done with every buffer
        done_in, done_dec = [], []
        for i in self.order:
            with torch.cuda.stream(self.s_in):
                self.blobs[i].copy_(self.pinned_in[i], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(self.s_in)
            done_in.append(ev)
        for j, i in enumerate(self.order):
            stream.wait_event(done_in[j])
            decode(self.descs[i], self.blobs[i], self.views[i], stream)
            ev = torch.cuda.Event()
            ev.record(stream)
            done_dec.append(ev)
        for j, i in enumerate(self.order):
            self.s_out.wait_event(done_dec[j])
            o, n = self.offsets[i], self.descs[i].n
            with torch.cuda.stream(self.s_out):
                self.host_out[o:o + n].copy_(self.views[i], non_blocking=True)
        stream.wait_stream(self.s_out)
