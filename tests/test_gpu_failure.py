"""Failure detection without a GPU fault: every kernel's waits on its
asynchronous copies are bounded; a wait that gives up reports
LWC_DEVICE_TIMEOUT through the caller's status word and the kernel returns, so
the context stays usable. lwc_selftest_bounded_wait runs that wait on an
mbarrier phase that nothing completes (no copy, no trap, no fault)."""
import numpy as np
import pytest
import torch

import synth
from decode_dfloat11_b200 import build as lwc_build
from decode_dfloat11_b200 import lwc

pytestmark = pytest.mark.gpu

LWC_DEVICE_TIMEOUT = lwc.LWC_DEVICE_TIMEOUT


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    lwc_build.build()
    return lwc.load()


@pytest.mark.parametrize("polls", [1, 64, 4096])
def test_wait_that_nothing_completes_reports_timeout(polls):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lwc.lwc_selftest_bounded_wait(status, polls, arrive=False)
    torch.cuda.synchronize()
    assert int(status.item()) == LWC_DEVICE_TIMEOUT


def test_completed_wait_reports_nothing_and_context_stays_usable():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lwc.lwc_selftest_bounded_wait(status, 4096, arrive=False)
    lwc.lwc_selftest_bounded_wait(status, 4096, arrive=False)
    torch.cuda.synchronize()
    assert int(status.item()) == LWC_DEVICE_TIMEOUT
    status.zero_()
    lwc.lwc_selftest_bounded_wait(status, 4096, arrive=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # after the timed-out waits the same context decodes exactly
    w = synth.as_u16(synth.normal_bf16((100_003,), seed=11, sigma=0.02, outlier_frac=1e-3))
    for enc, dec in ((lwc.lwc_encode_dfloat11, lwc.lwc_decode_dfloat11_checked),
                     (lwc.lwc_encode_codebook, lwc.lwc_decode_codebook_checked)):
        d, b = enc(w)
        out = torch.empty(w.size, dtype=torch.int16, device="cuda")
        dec(d, torch.from_numpy(b).to("cuda"), out, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert np.array_equal(out.cpu().numpy().view(np.uint16), w)
