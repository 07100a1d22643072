"""The no-allocation DFloat11 device encoder (lwc_encode_dfloat11_device_noalloc),
through the C ABI, against the two-call device encoder with a caller
workspace: two calls in a row on different tensors must each give the
workspace path's blob byte for byte (the second call also shows that the
first call's leftovers in the shared scratch array do not leak into it), and
the second call must not change the device's free memory.

Collected last on purpose (file name), and independent of the other test
files, so it passes alone in a fresh process and after the whole suite."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from decode_dfloat11_b200 import build as lwc_build
from decode_dfloat11_b200 import lwc

pytestmark = pytest.mark.gpu

MAX_N = 1 << 30


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    lwc_build.build()
    return lwc.load()


def with_workspace(src, n, **params):
    work_bytes = lwc.lwc_encode_device_workspace_bytes(n)
    work = torch.empty(work_bytes, dtype=torch.uint8, device="cuda")
    d = lwc.lwc_encode_dfloat11_device_plan(src, n, work, work_bytes, **params)
    blob = torch.empty(d.total_bytes, dtype=torch.uint8, device="cuda")
    d = lwc.lwc_encode_device_write(src, n, work, work_bytes, blob, blob.numel())
    return d, blob.cpu().numpy()


def test_noalloc_matches_workspace_encoder_on_two_calls_in_a_row():
    # a larger tensor first, then a smaller one with other parameters
    a = synth.normal_bf16((3_000_017,), seed=71, sigma=0.02, outlier_frac=1e-3, device="cuda")
    b = synth.normal_bf16((123_457,), seed=72, sigma=0.005, outlier_frac=1e-2, device="cuda")
    cases = [(a, {}), (b, dict(chunk_bytes=20, threads_per_block=128))]
    expected = [with_workspace(t, t.numel(), **p) for t, p in cases]
    outs = [torch.full((d.total_bytes + 4096,), 0x77, dtype=torch.uint8, device="cuda") for d, _ in expected]
    decoded = [torch.empty(t.numel(), dtype=torch.int16, device="cuda") for t, _ in cases]
    torch.cuda.synchronize()
    for i, ((t, params), (d_ref, blob_ref), out, dec) in enumerate(zip(cases, expected, outs, decoded)):
        free_before = torch.cuda.mem_get_info()[0]
        d = lwc.lwc_encode_dfloat11_device_noalloc(t, t.numel(), out, out.numel(), **params)
        torch.cuda.synchronize()
        if i == 1:   # the first call may load the library's device code (and its scratch array)
            assert torch.cuda.mem_get_info()[0] == free_before
        assert d.as_dict() == d_ref.as_dict()
        got = out.cpu().numpy()
        assert np.array_equal(got[:d.total_bytes], blob_ref), i
        assert (got[d.total_bytes:] == 0x77).all()   # nothing written past the blob
        # and it decodes back to the source
        lwc.lwc_decode_dfloat11(d, out, dec)
        torch.cuda.synchronize()
        assert torch.equal(dec, t.view(torch.int16))


def test_noalloc_rejects_oversized_tensors_and_short_blobs():
    with pytest.raises(lwc.LwcError) as e:
        lwc.lwc_encode_dfloat11_device_noalloc(0x1000, MAX_N + 1, 0x2000, 1 << 40)
    assert e.value.status == 4 and "maximum" in str(e.value)
    t = synth.normal_bf16((50_000,), seed=73, sigma=0.02, device="cuda")
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    L = lwc.load()
    desc = lwc.lwc_desc()
    st = L.lwc_encode_dfloat11_device_noalloc(t.data_ptr(), t.numel(), None, small.data_ptr(), small.numel(),
                                              ctypes.byref(desc), None)
    assert st == 1 and desc.total_bytes > small.numel()   # the plan says how much is needed
    blob = torch.empty(desc.total_bytes, dtype=torch.uint8, device="cuda")
    d = lwc.lwc_encode_dfloat11_device_noalloc(t, t.numel(), blob, blob.numel())
    torch.cuda.synchronize()
    assert np.array_equal(blob.cpu().numpy(), lwc.lwc_encode_dfloat11(synth.as_u16(t))[1])
    assert d.total_bytes == desc.total_bytes
