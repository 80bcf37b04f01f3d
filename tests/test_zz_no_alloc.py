"""lf_lora_shrink_expand_noalloc: the shrink/expand entry point for callers that
cannot allocate device memory (for example a serving loop that reserved all GPU
memory at start-up, or a latency-critical path that cannot afford cudaMalloc's
implicit synchronisation).  It takes no workspace; the library keeps the routing
scratch in a fixed device array.

Checked here through the C ABI against the workspace entry point, on calls in a row
that alternate between batch shapes (a few tokens per adapter, which takes the fused
single-launch GEMV kernel, and many tokens per adapter, which takes the separate
shrink and expand kernels), so stale scratch contents from an earlier call would show,
with the tolerance the apply parity tests use.  The file name
sorts last so a run that stops at the first failure has run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from post_hoc_rank_b200 import api, build, synth
from post_hoc_rank_b200 import loraforge as lf
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available()


def batch(T, n, d_in, d_out, seed):
    g = np.random.default_rng(seed)
    ranks = g.integers(1, 65, size=n).astype(np.int64)
    ids = synth.zipf_ids(T, n, 1.0, (40, seed))
    ids[g.random(T) < 0.1] = -1
    offA = np.concatenate([[0], np.cumsum(ranks * d_in)])
    offB = np.concatenate([[0], np.cumsum(ranks * d_out)])
    dev = "cuda"
    return dict(
        x=synth.normal_bf16((T, d_in), (40, seed, 1)).to(dev),
        y0=synth.normal_bf16((T, d_out), (40, seed, 2)).to(dev),
        ids=torch.from_numpy(ids).to(dev), n=n,
        ranks=torch.from_numpy(ranks.astype(np.int32)).to(dev),
        offA=torch.from_numpy(offA[:-1]).to(dev), offB=torch.from_numpy(offB[:-1]).to(dev),
        Ap=synth.normal_bf16((int(offA[-1]),), (40, seed, 3), std=d_in ** -0.5).to(dev),
        Bt=synth.normal_bf16((int(offB[-1]),), (40, seed, 4), std=d_out ** -0.5).to(dev))


def with_workspace(b, scale):
    y = b["y0"].clone()
    api.shrink_expand(b["x"], y, b["ids"], b["ranks"], b["offA"], b["offB"], b["Ap"], b["Bt"], scale)
    assert lf.lf_get_device_status() == 0
    return y


def without_workspace(b, scale):
    """Call the no-allocation entry point directly through the C ABI."""
    y = b["y0"].clone()
    T, d_in = b["x"].shape
    d_out = y.shape[1]
    st = lf.lib().lf_lora_shrink_expand_noalloc(
        T, d_in, d_out, b["x"].data_ptr(), y.data_ptr(), b["ids"].data_ptr(), b["n"], b["ranks"].data_ptr(),
        b["offA"].data_ptr(), b["offB"].data_ptr(), b["Ap"].data_ptr(), b["Bt"].data_ptr(),
        b["Ap"].numel(), b["Bt"].numel(), ctypes.c_float(scale), None,
        torch.cuda.current_stream().cuda_stream)
    assert st == 0
    assert lf.lf_get_device_status() == 0
    return y


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    many = batch(300, 37, 4096, 1024, seed=1)     # > 8 tokens per adapter: shrink + expand kernels
    few = batch(64, 37, 4096, 1024, seed=3)       # <= 8 tokens per adapter: fused GEMV kernel
    many2 = batch(77, 5, 1024, 2048, seed=2)
    few2 = batch(32, 16, 1024, 2048, seed=4)
    assert few["x"].shape[0] <= 8 * few["n"] and few2["x"].shape[0] <= 8 * few2["n"]
    assert many["x"].shape[0] > 8 * many["n"] and many2["x"].shape[0] > 8 * many2["n"]
    for b, scale in ((many, 0.5), (few, 1.5), (many2, 2.0), (few2, 0.75)):
        ref = with_workspace(b, scale)
        got = without_workspace(b, scale)
        delta_ref = (ref.float() - b["y0"].float()).abs().max().item()
        diff = (got.float() - ref.float()).abs().max().item()
        assert diff <= G.APPLY_TOL * max(ref.float().abs().max().item(), 1e-30)
        assert delta_ref > 0.0                       # the batch really touched y
        unrouted = b["ids"] < 0
        assert torch.equal(got[unrouted], b["y0"][unrouted])


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = lf.lib()
    big_T = lf.NOALLOC_MAX_TOKENS + 1
    st = L.lf_lora_shrink_expand_noalloc(big_T, 64, 64, 16, 16, 16, 2, 16, 16, 16, 16, 16, 1024, 1024,
                                         ctypes.c_float(1.0), None, None)
    assert st == 4  # LF_ERR_WORKSPACE, nothing launched
    st = L.lf_lora_shrink_expand_noalloc(8, 64, 64, 16, 16, 16, lf.NOALLOC_MAX_ADAPTERS + 1, 16, 16, 16, 16, 16,
                                         1024, 1024, ctypes.c_float(1.0), None, None)
    assert st == 4
