"""GPU parity of lf_lora_shrink_expand (routing + shrink/expand) against the fp64
oracle on the same bf16 bytes."""
import numpy as np
import pytest
import torch

from oracle import apply as OP
from post_hoc_rank_b200 import api, build, synth
from post_hoc_rank_b200 import loraforge as lf
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available()


def make_pools(ranks, d_in, d_out, key, std_a=None, std_b=None):
    """Packed bf16 pools (A' k x d_in, B'^T k x d_out per adapter), N(0, 1/d) entries."""
    ranks = np.asarray(ranks, dtype=np.int64)
    offA = np.concatenate([[0], np.cumsum(ranks * d_in)])
    offB = np.concatenate([[0], np.cumsum(ranks * d_out)])
    Ap = synth.normal_bf16((max(int(offA[-1]), 8),), key + (0,), std=std_a or d_in ** -0.5)
    Bt = synth.normal_bf16((max(int(offB[-1]), 8),), key + (1,), std=std_b or d_out ** -0.5)
    return offA, offB, Ap, Bt


def run_apply(x, y0, ids, ranks, offA, offB, Ap, Bt, scale, seg=False):
    dev = "cuda"
    T = x.shape[0]
    n = len(ranks)
    y = y0.clone().to(dev)
    seg_out = torch.full((2 + 3 * min(T, n) + T,), -7, dtype=torch.int32, device=dev) if seg else None
    api.shrink_expand(x.to(dev), y, torch.from_numpy(np.asarray(ids, np.int32)).to(dev),
                      torch.from_numpy(np.asarray(ranks, np.int32)).to(dev),
                      torch.from_numpy(np.asarray(offA[:-1], np.int64)).to(dev),
                      torch.from_numpy(np.asarray(offB[:-1], np.int64)).to(dev),
                      Ap.to(dev), Bt.to(dev), scale, seg_out=seg_out)
    st = lf.lf_get_device_status()
    return y.cpu(), (seg_out.cpu().numpy() if seg else None), st


def oracle_y(x, y0, ids, ranks, offA, offB, Ap, Bt, scale):
    return OP.lora_apply(x.float().numpy(), y0.float().numpy(), ids, ranks, offA[:-1], offB[:-1],
                         Ap.float().numpy(), Bt.float().numpy(), scale)


def assert_close(y_gpu, y_orc):
    d = np.abs(y_gpu.float().numpy().astype(np.float64) - y_orc).max()
    assert d <= G.APPLY_TOL * max(np.abs(y_orc).max(), 1e-30), (d, np.abs(y_orc).max())


def check_routing(seg, ids, n):
    segs_o, perm_o = OP.route(ids, n)
    nseg, nval = int(seg[0]), int(seg[1])
    assert nseg == len(segs_o) and nval == len(perm_o)
    assert seg[2:2 + 3 * nseg].reshape(-1, 3).tolist() == segs_o.tolist()
    assert seg[2 + 3 * nseg:2 + 3 * nseg + nval].tolist() == perm_o.tolist()


def test_tiny_apply_and_routing():
    T, n, d, k = 64, 4, 256, 4
    ids = synth.uniform_ids(T, n, (1, 0))
    offA, offB, Ap, Bt = make_pools([k] * n, d, d, (1, 1))
    x = synth.normal_bf16((T, d), (1, 2))
    y0 = torch.zeros(T, d, dtype=torch.bfloat16)
    y, seg, st = run_apply(x, y0, ids, [k] * n, offA, offB, Ap, Bt, 2.0, seg=True)
    assert st == 0
    assert_close(y, oracle_y(x, y0, ids, [k] * n, offA, offB, Ap, Bt, 2.0))
    check_routing(seg, ids, n)


@pytest.mark.parametrize("d_in,d_out", [(4096, 1024), (1024, 14336), (3584, 512)])
@pytest.mark.parametrize("n", [37, 64])   # 37: split shrink/expand path, 64: fused decode path
def test_ragged_ranks_zipf_with_unrouted_tokens(d_in, d_out, n):
    T = 300
    g = np.random.default_rng(5)
    ranks = g.integers(1, 65, size=n)
    ids = synth.zipf_ids(T, n, 1.0, (2, d_in))
    ids[g.random(T) < 0.1] = -1
    offA, offB, Ap, Bt = make_pools(ranks, d_in, d_out, (2, d_out))
    x = synth.normal_bf16((T, d_in), (2, 3))
    y0 = synth.normal_bf16((T, d_out), (2, 4))
    y, seg, st = run_apply(x, y0, ids, ranks, offA, offB, Ap, Bt, 0.5, seg=True)
    assert st == 0
    check_routing(seg, ids, n)
    # unrouted rows are untouched, bit for bit
    assert torch.equal(y[torch.from_numpy(ids < 0)], y0[torch.from_numpy(ids < 0)])
    # the LoRA delta itself against the oracle (y0 = 0 measures the delta alone)
    yz, _, _ = run_apply(x, torch.zeros_like(y0), ids, ranks, offA, offB, Ap, Bt, 0.5)
    assert_close(yz, oracle_y(x, torch.zeros_like(y0), ids, ranks, offA, offB, Ap, Bt, 0.5))


def test_bad_index_latches_error_and_skips_token():
    T, n, d = 16, 3, 256
    ids = np.array([0, 1, 2, 5, -3] + [1] * 11, dtype=np.int32)
    offA, offB, Ap, Bt = make_pools([2, 3, 4], d, d, (3, 0))
    x = synth.normal_bf16((T, d), (3, 1))
    y0 = synth.normal_bf16((T, d), (3, 2))
    y, _, st = run_apply(x, y0, ids, [2, 3, 4], offA, offB, Ap, Bt, 1.0)
    assert st == 3  # LF_ERR_BAD_INDEX
    assert torch.equal(y[3], y0[3]) and torch.equal(y[4], y0[4])


def test_scale_zero_leaves_y():
    T, n, d = 40, 5, 512
    ids = synth.uniform_ids(T, n, (4, 0))
    offA, offB, Ap, Bt = make_pools([3] * n, d, d, (4, 1))
    x = synth.normal_bf16((T, d), (4, 2))
    y0 = synth.normal_bf16((T, d), (4, 3))
    y, _, st = run_apply(x, y0, ids, [3] * n, offA, offB, Ap, Bt, 0.0)
    assert st == 0 and torch.equal(y, y0)


@pytest.mark.parametrize("k", [16, 64])
def test_prefill_segments(k):
    # 4 requests x 512 tokens, request i -> adapter i; Qwen-like widths
    T, n, d_in, d_out = 2048, 4, 3584, 18944
    ids = np.repeat(np.arange(n, dtype=np.int32), 512)
    offA, offB, Ap, Bt = make_pools([k] * n, d_in, d_out, (5, k))
    x = synth.normal_bf16((T, d_in), (5, 1))
    y0 = torch.zeros(T, d_out, dtype=torch.bfloat16)
    y, seg, st = run_apply(x, y0, ids, [k] * n, offA, offB, Ap, Bt, 2.0, seg=True)
    assert st == 0
    check_routing(seg, ids, n)
    assert_close(y, oracle_y(x, y0, ids, [k] * n, offA, offB, Ap, Bt, 2.0))


@pytest.mark.parametrize("widths", [[1000], [512, 256, 264]])
def test_tensor_core_x_by_tma_equals_gather(widths):
    """Segments whose tokens are consecutive rows of x load the shrink's x stages with one
    TMA copy each; the same segments interleaved (order inside each segment kept) are
    gathered row by row.  The tiles hold the same rows in the same order, so y is equal
    bit for bit, and both match the oracle.  Cases: partial tiles followed by another
    adapter's rows and by the end of x, d_in = 3000 (two splits, the last stage past
    d_in), one slice (N <= 64) and three (N <= 256)."""
    adapters = [2, 0, 3, 1, 4]
    lens = [300, 129, 64, 1000, 200]
    n, d_in = 5, 3000
    ids = np.concatenate([np.full(c, a, dtype=np.int32) for a, c in zip(adapters, lens)])
    T = len(ids)
    sl, y_ld = make_slices(widths, n, d_in, (15, 1, len(widths)))
    x = synth.normal_bf16((T, d_in), (15, 2))
    y0 = synth.normal_bf16((T, y_ld), (15, 3))
    y, _, st = run_slices(x, y0, ids, sl, 0.75)
    assert st == 0
    check_slices(y, y0, oracle_slices(x, y0, ids, sl, 0.75), sl, ids)
    # interleave: position p takes the next token (in order) of adapter labels[p]
    labels = np.random.default_rng(15).permutation(ids)
    pos = np.empty(T, dtype=np.int64)
    for a in adapters:
        pos[np.flatnonzero(ids == a)] = np.flatnonzero(labels == a)
    inv = torch.from_numpy(np.argsort(pos))
    xi, y0i = x[inv], y0[inv]
    yi, _, st = run_slices(xi, y0i, labels, sl, 0.75)
    assert st == 0
    assert torch.equal(yi[torch.from_numpy(pos)], y)


def test_empty_batch_and_all_unrouted():
    d = 256
    offA, offB, Ap, Bt = make_pools([2], d, d, (6, 0))
    x = synth.normal_bf16((8, d), (6, 1)); y0 = synth.normal_bf16((8, d), (6, 2))
    y, seg, st = run_apply(x, y0, [-1] * 8, [2], offA, offB, Ap, Bt, 1.0, seg=True)
    assert st == 0 and torch.equal(y, y0) and seg[0] == 0 and seg[1] == 0
    y, _, st = run_apply(x[:0], y0[:0], [], [2], offA, offB, Ap, Bt, 1.0)
    assert st == 0 and y.shape == (0, d)


def test_routing_of_long_mixed_batch():
    # > 4 chunks of the routing block: long runs (prefill requests), single tokens
    # (decode requests) and unrouted tokens interleaved; the segment table and the
    # permutation must equal the stable argsort bit for bit
    g = np.random.default_rng(17)
    n, d = 100, 256
    parts = []
    while sum(len(p) for p in parts) < 5000:
        if g.random() < 0.3:
            parts.append(np.full(int(g.integers(20, 400)), int(g.integers(0, n)), dtype=np.int32))
        else:
            parts.append(g.integers(-1, n, size=int(g.integers(1, 40))).astype(np.int32))
    ids = np.concatenate(parts)[:5000]
    T = len(ids)
    ranks = g.integers(1, 17, size=n)
    offA, offB, Ap, Bt = make_pools(ranks, d, d, (7, 0))
    x = synth.normal_bf16((T, d), (7, 1))
    y0 = torch.zeros(T, d, dtype=torch.bfloat16)
    y, seg, st = run_apply(x, y0, ids, ranks, offA, offB, Ap, Bt, 1.0, seg=True)
    assert st == 0
    check_routing(seg, ids, n)
    assert_close(y, oracle_y(x, y0, ids, ranks, offA, offB, Ap, Bt, 1.0))


def make_slices(widths, n, d_in, key, rank_hi=65):
    """Per-slice pools with ragged ranks; slices laid out in y with an 8-column gap each."""
    g = np.random.default_rng(key[-1])
    out, y_off = [], 0
    for s, d_out in enumerate(widths):
        ranks = g.integers(1, rank_hi, size=n)
        offA, offB, Ap, Bt = make_pools(ranks, d_in, d_out, key + (s,))
        out.append(dict(d_out=d_out, y_off=y_off, ranks=ranks, offA=offA, offB=offB, Ap=Ap, Bt=Bt))
        y_off += d_out + 8
    return out, y_off


def run_slices(x, y0, ids, sl, scale, adapter_scale=None, seg=False):
    dev = "cuda"
    T = x.shape[0]
    n = len(sl[0]["ranks"])
    y = y0.clone().to(dev)
    keep = []
    tup = []
    for s in sl:
        t = (s["d_out"], s["y_off"], torch.from_numpy(np.asarray(s["ranks"], np.int32)).to(dev),
             torch.from_numpy(np.asarray(s["offA"][:-1], np.int64)).to(dev),
             torch.from_numpy(np.asarray(s["offB"][:-1], np.int64)).to(dev), s["Ap"].to(dev), s["Bt"].to(dev))
        keep.append(t)
        tup.append(t)
    seg_out = torch.full((2 + 3 * min(T, n) + T,), -7, dtype=torch.int32, device=dev) if seg else None
    asc = torch.from_numpy(np.asarray(adapter_scale, np.float32)).to(dev) if adapter_scale is not None else None
    api.shrink_expand_slices(x.to(dev), y, torch.from_numpy(np.asarray(ids, np.int32)).to(dev), tup, scale,
                             adapter_scale=asc, seg_out=seg_out)
    st = lf.lf_get_device_status()
    return y.cpu(), (seg_out.cpu().numpy() if seg else None), st


def oracle_slices(x, y0, ids, sl, scale, adapter_scale=None):
    tup = [(s["d_out"], s["y_off"], s["ranks"], s["offA"][:-1], s["offB"][:-1], s["Ap"].float().numpy(),
            s["Bt"].float().numpy()) for s in sl]
    return OP.lora_apply_slices(x.float().numpy(), y0.float().numpy(), ids, tup, scale, adapter_scale)


def bf16_half_ulp(v):
    """Half a bf16 ulp at |v| (8 significant bits): the error of the one rounding of y."""
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -126)))
    return 2.0 ** (e - 8)


def check_slices(y, y0, want, sl, ids):
    """Per slice: |y - want| within APPLY_TOL of the slice's largest LoRA delta, after
    allowing the one bf16 rounding of y = y0 + s B't (half an ulp of |want|); columns
    outside the slices and unrouted rows bit-equal to y0."""
    yv = y.float().numpy().astype(np.float64)
    covered = np.zeros(y.shape[1], dtype=bool)
    for s in sl:
        c = slice(s["y_off"], s["y_off"] + s["d_out"])
        d = np.maximum(np.abs(yv[:, c] - want[:, c]) - bf16_half_ulp(want[:, c]), 0.0).max()
        delta = np.abs(want[:, c] - y0.float().numpy()[:, c]).max()
        assert d <= G.APPLY_TOL * max(delta, 1e-30), (s["d_out"], d, delta)
        covered[c] = True
    assert torch.equal(y[:, torch.from_numpy(~covered)], y0[:, torch.from_numpy(~covered)])   # gaps untouched
    assert torch.equal(y[torch.from_numpy(ids < 0)], y0[torch.from_numpy(ids < 0)])           # unrouted rows


@pytest.mark.parametrize("regime", ["decode", "gemv", "tensor_core"])
def test_slices_match_oracle(regime):
    # q/k/v-like slices sharing x; per-adapter scales; the three execution regimes:
    # token-parallel (T <= 8n), sorted GEMV items (short segments), tcgen05 tiles
    d_in = 512
    if regime == "decode":
        T, n = 96, 32
        ids = synth.zipf_ids(T, n, 1.0, (8, 0))
    elif regime == "gemv":
        T, n = 300, 37
        ids = synth.zipf_ids(T, n, 1.0, (8, 1))
    else:
        T, n = 1024, 4
        ids = np.repeat(np.arange(n, dtype=np.int32), 256)
    ids = ids.copy()
    ids[np.random.default_rng(3).random(T) < 0.05] = -1
    sl, y_ld = make_slices([512, 128, 256], n, d_in, (8, 2, T))
    x = synth.normal_bf16((T, d_in), (8, 3, T))
    y0 = synth.normal_bf16((T, y_ld), (8, 4, T))
    asc = 0.5 + np.arange(n) / n
    y, seg, st = run_slices(x, y0, ids, sl, 1.0, adapter_scale=asc, seg=True)
    assert st == 0
    check_routing(seg, ids, n)
    check_slices(y, y0, oracle_slices(x, y0, ids, sl, 1.0, asc), sl, ids)


def test_one_slice_call_equals_projection_call():
    # lf_lora_shrink_expand is the one-slice case of the slice entry point: same bits
    T, n, d_in, d_out = 2048, 4, 1024, 512
    ids = np.repeat(np.arange(n, dtype=np.int32), 512)
    offA, offB, Ap, Bt = make_pools([16, 24, 8, 64], d_in, d_out, (9, 0))
    x = synth.normal_bf16((T, d_in), (9, 1))
    y0 = synth.normal_bf16((T, d_out), (9, 2))
    y1, _, st1 = run_apply(x, y0, ids, [16, 24, 8, 64], offA, offB, Ap, Bt, 0.75)
    sl = [dict(d_out=d_out, y_off=0, ranks=np.array([16, 24, 8, 64]), offA=offA, offB=offB, Ap=Ap, Bt=Bt)]
    y2, _, st2 = run_slices(x, y0, ids, sl, 0.75)
    assert st1 == 0 and st2 == 0
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("regime", ["decode", "gemv", "tensor_core"])
@pytest.mark.parametrize("diagonal", [True, False])
def test_sigma_sandwich_matches_oracle(regime, diagonal):
    # jointly compressed adapters: shared V^T, U^T and a Sigma_a per adapter
    d_in, d_out, r = 512, 1024, 24
    if regime == "decode":
        T, n = 96, 32
        ids = synth.zipf_ids(T, n, 1.0, (10, 0))
    elif regime == "gemv":
        T, n = 300, 37
        ids = synth.zipf_ids(T, n, 1.0, (10, 1))
    else:
        T, n = 1024, 4
        ids = np.repeat(np.arange(n, dtype=np.int32), 256)
    ids = ids.copy()
    ids[np.random.default_rng(11).random(T) < 0.05] = -1
    Vt = synth.normal_bf16((r, d_in), (10, 2), std=d_in ** -0.5)
    Ut = synth.normal_bf16((r, d_out), (10, 3), std=d_out ** -0.5)
    g = np.random.default_rng(12)
    sig = (g.standard_normal((n, r)) if diagonal else g.standard_normal((n, r, r)) / np.sqrt(r)).astype(np.float32)
    x = synth.normal_bf16((T, d_in), (10, 4))
    y0 = torch.zeros(T, d_out, dtype=torch.bfloat16)
    dev = "cuda"
    y = y0.clone().to(dev)
    ws = api.workspace(lf.lf_apply_workspace_size(T, n), dev)
    lf.lf_lora_sigma_sandwich(x.to(dev), y, torch.from_numpy(ids).to(dev), n, Vt.to(dev), Ut.to(dev),
                              torch.from_numpy(sig).to(dev), diagonal, 1.5, ws)
    assert lf.lf_get_device_status() == 0
    want = OP.sigma_sandwich_apply(x.float().numpy(), y0.float().numpy(), ids, Vt.float().numpy(),
                                   Ut.float().numpy(), sig.astype(np.float64), diagonal, 1.5)
    assert_close(y.cpu(), want)
    assert torch.equal(y.cpu()[torch.from_numpy(ids < 0)], y0[torch.from_numpy(ids < 0)])


def _slice_tensors(sl, dev="cuda"):
    """lf_slice records and the device tensors they point into (keep both alive)."""
    tens = [(s["d_out"], s["y_off"], torch.from_numpy(np.asarray(s["ranks"], np.int32)).to(dev),
             torch.from_numpy(np.asarray(s["offA"][:-1], np.int64)).to(dev),
             torch.from_numpy(np.asarray(s["offB"][:-1], np.int64)).to(dev), s["Ap"].to(dev), s["Bt"].to(dev))
            for s in sl]
    return [lf.make_slice(*t) for t in tens], tens


def test_routing_once_serves_every_projection():
    """lf_route_tokens + routed calls give the same bits as unrouted calls, for projections
    with different slice counts on one workspace (segments for both GEMV and tensor-core items)."""
    T, n, d_in = 1500, 6, 256
    ids = np.concatenate([np.repeat(np.arange(4, dtype=np.int32), 300), synth.zipf_ids(300, n, 1.0, (12, 0))])
    ids[np.random.default_rng(12).random(T) < 0.03] = -1
    ids_d = torch.from_numpy(ids).cuda()
    x = synth.normal_bf16((T, d_in), (12, 1)).cuda()
    projs = [make_slices([256], n, d_in, (12, 2)), make_slices([128, 64, 64], n, d_in, (12, 3))]
    ws = api.workspace(lf.lf_apply_slices_workspace_size(T, n, 3), "cuda")
    lf.lf_route_tokens(ids_d, n, ws)
    for p, (sl, y_ld) in enumerate(projs):
        y0 = synth.normal_bf16((T, y_ld), (12, 4, p)).cuda()
        keep, _alive = _slice_tensors(sl)
        y_ref = y0.clone()
        ws_ref = api.workspace(lf.lf_apply_slices_workspace_size(T, n, len(sl)), "cuda")
        lf.lf_lora_shrink_expand_slices(x, y_ref, ids_d, n, keep, 1.25, ws_ref)
        y = y0.clone()
        lf.lf_lora_shrink_expand_slices_routed(x, y, ids_d, n, keep, 1.25, ws)
        assert lf.lf_get_device_status() == 0
        assert torch.equal(y, y_ref), p
        check_slices(y.cpu(), y0.cpu(), oracle_slices(x.cpu(), y0.cpu(), ids, sl, 1.25), sl, ids)


def test_routed_call_without_matching_routing_applies_nothing():
    T, n, d_in = 600, 3, 128
    ids = np.repeat(np.arange(n, dtype=np.int32), 200)
    ids_d = torch.from_numpy(ids).cuda()
    x = synth.normal_bf16((T, d_in), (13, 1)).cuda()
    sl, y_ld = make_slices([128], n, d_in, (13, 2))
    keep, _alive = _slice_tensors(sl)
    y0 = synth.normal_bf16((T, y_ld), (13, 3)).cuda()
    # a fresh (zeroed) workspace: no routing pass ever ran on it
    ws = torch.zeros(lf.lf_apply_slices_workspace_size(T, n, 1), dtype=torch.uint8, device="cuda")
    y = y0.clone()
    lf.lf_lora_shrink_expand_slices_routed(x, y, ids_d, n, keep, 1.0, ws)
    assert lf.lf_get_device_status() == 1   # LF_ERR_INVALID_ARG, latched on the device
    assert torch.equal(y, y0)
    # routing written for another batch shape (fewer tokens) is not reused either
    lf.lf_route_tokens(ids_d[:300], n, ws)
    assert lf.lf_get_device_status() == 0
    lf.lf_lora_shrink_expand_slices_routed(x, y, ids_d, n, keep, 1.0, ws)
    assert lf.lf_get_device_status() == 1
    assert torch.equal(y, y0)


@pytest.mark.parametrize("d_in,widths", [
    (256, [256, 128]),
    (1544, [264]),
    (2056, [4000, 1024, 1016]),   # q/k/v-like slices
    (4104, [14344]),              # gate-like widths, one 16384-column chunk
])
def test_routed_call_in_decode_regime(d_in, widths):
    """T <= 8 n: the token-parallel kernel indexes the adapter of every token, so a routed
    call gives the unrouted call's bits whatever the routing tables hold; both match the
    oracle.  Zipf ids give an adapter more than one GEMV item of tokens; 5% unrouted."""
    T, n = 300, 64
    ids = synth.zipf_ids(T, n, 1.0, (14, d_in)).copy()
    ids[np.random.default_rng(14).random(T) < 0.05] = -1
    assert np.bincount(ids[ids >= 0]).max() > 8
    ids_d = torch.from_numpy(ids).cuda()
    x = synth.normal_bf16((T, d_in), (14, 1, d_in))
    sl, y_ld = make_slices(widths, n, d_in, (14, 2, d_in))
    keep, _alive = _slice_tensors(sl)
    y0 = synth.normal_bf16((T, y_ld), (14, 3, d_in))
    asc = torch.from_numpy((0.5 + np.arange(n) / n).astype(np.float32)).cuda()
    ws = api.workspace(lf.lf_apply_slices_workspace_size(T, n, len(sl)), "cuda")
    lf.lf_route_tokens(ids_d, n, ws)
    y = y0.cuda()
    lf.lf_lora_shrink_expand_slices_routed(x.cuda(), y, ids_d, n, keep, 1.0, ws, adapter_scale=asc)
    y_ref = y0.cuda()
    lf.lf_lora_shrink_expand_slices(x.cuda(), y_ref, ids_d, n, keep, 1.0,
                                    api.workspace(lf.lf_apply_slices_workspace_size(T, n, len(sl)), "cuda"),
                                    adapter_scale=asc)
    assert lf.lf_get_device_status() == 0
    assert torch.equal(y, y_ref)
    check_slices(y.cpu(), y0, oracle_slices(x, y0, ids, sl, 1.0, asc.cpu().numpy()), sl, ids)


def test_mixed_batch_with_many_resident_adapters_reaches_tensor_cores():
    """With 1024 resident adapters a batch of more than 8 tokens per resident adapter is
    routed per segment: 17 prefill requests of 512 tokens go to the tensor-core tiles,
    a 48-token request and the decode tokens to the token-parallel kernel in routing
    order, in one call; the result matches the oracle and the routing equals the
    stable argsort."""
    n, d_in, d_out = 1024, 1024, 2048
    g = np.random.default_rng(18)
    ranks = g.integers(1, 17, size=n)
    dec = synth.zipf_ids(1024, n, 1.2, (18, 0))
    reqs = [np.full(512, a, np.int32) for a in g.choice(n, 17, replace=False)]
    ids = np.concatenate(reqs[:9] + [dec[:600], np.full(48, 33, np.int32)] + reqs[9:] + [dec[600:]]).astype(np.int32)
    ids[g.random(len(ids)) < 0.02] = -1
    T = len(ids)
    assert T > 8 * n
    offA, offB, Ap, Bt = make_pools(ranks, d_in, d_out, (18, 1))
    x = synth.normal_bf16((T, d_in), (18, 2))
    y0 = torch.zeros(T, d_out, dtype=torch.bfloat16)
    lf.lf_profile_reset(); lf.lf_profile_enable(True)
    y, seg, st = run_apply(x, y0, ids, ranks, offA, offB, Ap, Bt, 2.0, seg=True)
    lf.lf_profile_enable(False)
    ph = lf.lf_profile_read()
    assert st == 0
    for name in ("route", "shrink_tc", "expand_tc", "bgmv"):
        assert name in ph and ph[name][1] > 0, (name, ph)
    check_routing(seg, ids, n)
    assert_close(y, oracle_y(x, y0, ids, ranks, offA, offB, Ap, Bt, 2.0))
    assert torch.equal(y[torch.from_numpy(ids < 0)], y0[torch.from_numpy(ids < 0)])


def _layer_projections(T, n, key, d_h=512, d_kv=128, d_ffn=1368):
    """A small layer: q, k, v (one y, slices with gaps), o, gate and up (one y), down; x_h
    feeds q/k/v/gate/up, x_o feeds o, x_f feeds down.  Per projection: (x, y0, slice dict)."""
    x_h = synth.normal_bf16((T, d_h), key + (1,))
    x_o = synth.normal_bf16((T, d_h), key + (2,))
    x_f = synth.normal_bf16((T, d_ffn), key + (3,))
    out = []
    for gi, (x, widths) in enumerate([(x_h, [d_h, d_kv, d_kv]), (x_o, [d_h]), (x_h, [d_ffn, d_ffn]), (x_f, [d_h])]):
        sl, y_ld = make_slices(widths, n, x.shape[1], key + (4, gi))
        y0 = synth.normal_bf16((T, y_ld), key + (5, gi))
        out.append((x, y0, sl))
    return out


@pytest.mark.parametrize("regime", ["decode", "routed"])
def test_projections_call_matches_oracle(regime):
    """Seven projections of a layer (four inputs, four outputs, q/k/v and gate/up as slices
    of one y) in one lf_lora_shrink_expand_projections call: the same bits as one
    lf_lora_shrink_expand_slices call per projection, and the oracle per projection."""
    if regime == "decode":
        T, n = 200, 64
        ids = synth.zipf_ids(T, n, 1.0, (15, 0)).copy()
    else:   # T > 8 n: routed, segments long enough for the tensor-core tiles
        T, n = 1200, 16
        ids = np.repeat(np.arange(n, dtype=np.int32), T // n)
        ids[:300] = synth.zipf_ids(300, n, 1.0, (15, 1))
    ids[np.random.default_rng(15).random(T) < 0.05] = -1
    ids_d = torch.from_numpy(ids).cuda()
    layer = _layer_projections(T, n, (15, 2, T))
    asc = torch.from_numpy((0.5 + np.arange(n) / n).astype(np.float32)).cuda()
    projs, alive, ys, ys_ref = [], [], [], []
    for x, y0, sl in layer:
        xd = x.cuda()
        keep, tens = _slice_tensors(sl)
        alive += [xd, tens]
        y = y0.cuda()
        ys.append(y)
        for s in keep:
            projs.append(lf.make_projection(xd, y, s))
        y_ref = y0.cuda()
        lf.lf_lora_shrink_expand_slices(xd, y_ref, ids_d, n, keep, 1.0,
                                        api.workspace(lf.lf_apply_slices_workspace_size(T, n, len(keep)), "cuda"),
                                        adapter_scale=asc)
        ys_ref.append(y_ref)
    assert len(projs) == 7
    ws = api.workspace(lf.lf_apply_workspace_size(T, n), "cuda") if regime == "routed" else None
    l0 = lf.lf_launch_count()
    lf.lf_lora_shrink_expand_projections(T, ids_d, n, projs, 1.0, ws, adapter_scale=asc)
    launches = lf.lf_launch_count() - l0
    assert lf.lf_get_device_status() == 0
    if regime == "decode":
        assert launches == 1
    for (x, y0, sl), y, y_ref in zip(layer, ys, ys_ref):
        # one projection at a time against the per-slice call and the oracle
        assert torch.equal(y, y_ref)
        check_slices(y.cpu(), y0, oracle_slices(x, y0, ids, sl, 1.0, asc.cpu().numpy()), sl, ids)


def test_projections_call_host_checks():
    """Host errors come back before anything runs: a misaligned y, too many projections,
    a nonzero reserved field."""
    T, n = 64, 16
    ids_d = torch.from_numpy(synth.zipf_ids(T, n, 1.0, (16, 0))).cuda()
    (x, y0, sl), = _layer_projections(T, n, (16, 1))[1:2]
    keep, _alive = _slice_tensors(sl)
    xd, y = x.cuda(), y0.cuda()
    good = lf.make_projection(xd, y, keep[0])
    assert lf.lf_lora_shrink_expand_projections(T, ids_d, n, [good] * 9, 1.0, check=False) == 1
    bad = lf.make_projection(xd, y, keep[0])
    bad.y = bad.y + 2   # not 16-byte aligned
    assert lf.lf_lora_shrink_expand_projections(T, ids_d, n, [good, bad], 1.0, check=False) == 8   # LF_ERR_ALIGNMENT
    res = lf.make_projection(xd, y, keep[0])
    res.reserved = 1
    assert lf.lf_lora_shrink_expand_projections(T, ids_d, n, [res], 1.0, check=False) == 1
    torch.cuda.synchronize()
    assert torch.equal(y.cpu(), y0)


def test_rank_bound_leaves_out_the_rank64_expand():
    """A slice whose caller bounds its ranks by 16 (lf_slice.max_rank): the same bits with
    one launch fewer on the tensor-core path; an adapter above the bound latches
    LF_ERR_SHAPE and its rows keep y; a bound above 64 is a host error."""
    T, n, d_in, d_out = 1024, 4, 512, 384
    ids = np.repeat(np.arange(n, dtype=np.int32), T // n)
    ids_d = torch.from_numpy(ids).cuda()
    x = synth.normal_bf16((T, d_in), (17, 1)).cuda()
    y0 = synth.normal_bf16((T, d_out), (17, 2)).cuda()
    ws = api.workspace(lf.lf_apply_slices_workspace_size(T, n, 1), "cuda")

    def run(ranks, bound):
        offA, offB, Ap, Bt = make_pools(ranks, d_in, d_out, (17, 3, len(ranks)))
        sl = [dict(d_out=d_out, y_off=0, ranks=np.asarray(ranks), offA=offA, offB=offB, Ap=Ap, Bt=Bt)]
        keep, tens = _slice_tensors(sl)
        keep[0].max_rank = bound
        y = y0.clone()
        l0 = lf.lf_launch_count()
        st = lf.lf_lora_shrink_expand_slices(x, y, ids_d, n, keep, 1.0, ws, check=False)
        return st, y, lf.lf_launch_count() - l0, sl, tens

    st0, y_free, l_free, sl, _a = run([16, 8, 16, 12], 0)
    st1, y_bound, l_bound, _, _b = run([16, 8, 16, 12], 16)
    assert st0 == 0 and st1 == 0 and lf.lf_get_device_status() == 0
    assert torch.equal(y_free, y_bound) and l_bound == l_free - 1
    check_slices(y_bound.cpu(), y0.cpu(), oracle_slices(x.cpu(), y0.cpu(), ids, sl, 1.0), sl, ids)
    st2, y_bad, _, sl2, _c = run([16, 20, 8, 4], 16)
    assert st2 == 0 and lf.lf_get_device_status() == 2   # LF_ERR_SHAPE
    rows = torch.from_numpy(ids == 1)
    assert torch.equal(y_bad.cpu()[rows], y0.cpu()[rows])
    want = oracle_slices(x.cpu(), y0.cpu(), ids, sl2, 1.0)
    keep_rows = ids != 1   # the other adapters as usual
    check_slices(y_bad.cpu()[torch.from_numpy(keep_rows)], y0.cpu()[torch.from_numpy(keep_rows)], want[keep_rows],
                 sl2, ids[keep_rows])
    st3, _, _, _, _d = run([16, 8, 16, 12], 65)
    assert st3 == 1   # LF_ERR_INVALID_ARG before any launch
