"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every pipeline of the library waits on mbarriers with a bounded loop; a producer that
never arrives makes the wait give up, latch LF_ERR_TIMEOUT in the device error word
and return, instead of hanging the GPU.  lf_check_bounded_wait runs that exact wait
on a barrier nothing arrives at (no copy or MMA in flight), with a budget of a few
polls, so the timeout branch runs; the host then reads the latched status and the
context stays usable for the next call."""
import numpy as np
import pytest
import torch

from oracle import factor as OF
from post_hoc_rank_b200 import api, build, synth
from post_hoc_rank_b200 import loraforge as lf

pytestmark = pytest.mark.gpu

LF_ERR_TIMEOUT = 6


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available()


def test_bounded_wait_runs_out_and_latches_timeout():
    L = lf.lib()
    stream = torch.cuda.current_stream().cuda_stream
    assert lf.lf_get_device_status() == 0
    for polls in (0, 16, 256):
        assert L.lf_check_bounded_wait(polls, stream) == 0
        assert lf.lf_get_device_status() == LF_ERR_TIMEOUT
        assert lf.lf_get_device_status() == 0                 # read once, then cleared


def test_context_usable_after_timeout():
    L = lf.lib()
    assert L.lf_check_bounded_wait(8, torch.cuda.current_stream().cuda_stream) == 0
    assert lf.lf_get_device_status() == LF_ERR_TIMEOUT
    # the factor path still runs and matches the oracle afterwards
    lay, Bh, Ah = synth.tiny_fleet()
    F = api.tsqr(api.modules_from_layout(lay), Bh.cuda(), Ah.cuda())
    assert lf.lf_get_device_status() == 0
    Bn, An = synth.module_view(lay, Bh, Ah, 0)
    s, *_ = OF.spectrum_factor(Bn.numpy(), An.numpy())
    assert np.abs(F.sigma[0].cpu().numpy()[:len(s)] - s).max() <= 2e-5 * s[0]
