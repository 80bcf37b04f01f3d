"""Pins for oracle.apply: hand case, brute force, routing by bucket loop, invariants."""
import json
import os

import numpy as np
import pytest

from oracle import apply as AP
from tests.conftest import GOLDEN

GOLD = json.load(open(os.path.join(GOLDEN, "small_factors.json")))


@pytest.mark.parametrize("case", GOLD["apply"])
def test_apply_hand_case(case):
    y = AP.lora_apply(np.array(case["x"], float), np.array(case["y0"], float), case["ids"],
                      case["ranks"], [0], [0], np.array(case["A_pool"], float),
                      np.array(case["Bt_pool"], float), case["scale"])
    np.testing.assert_array_equal(y, np.array(case["y"], float))


def bucket_route(ids, n):
    buckets = [[] for _ in range(n)]
    for t, a in enumerate(ids):
        if a >= 0:
            buckets[a].append(t)
    segs, perm = [], []
    for a in range(n):
        if buckets[a]:
            segs.append((a, len(perm), len(buckets[a])))
            perm.extend(buckets[a])
    return segs, perm


@pytest.mark.parametrize("seed", range(5))
def test_route_matches_bucket_loop(seed):
    g = np.random.default_rng(seed)
    n = int(g.integers(1, 20))
    ids = g.integers(-1, n, size=int(g.integers(0, 300)))
    segs, perm = AP.route(ids, n)
    s2, p2 = bucket_route(ids.tolist(), n)
    assert [tuple(s) for s in segs.tolist()] == s2
    assert perm.tolist() == p2


def test_route_rejects_bad_ids():
    with pytest.raises(ValueError):
        AP.route([0, 3], 3)
    with pytest.raises(ValueError):
        AP.route([0, -2], 3)


def make_pools(g, n, d_in, d_out, ranks):
    offA = np.zeros(n, np.int64); offB = np.zeros(n, np.int64)
    ta = tb = 0
    for a in range(n):
        offA[a], offB[a] = ta, tb
        ta += ranks[a] * d_in; tb += ranks[a] * d_out
    return offA, offB, g.standard_normal(ta), g.standard_normal(tb)


@pytest.mark.parametrize("seed", range(4))
def test_apply_matches_dense_delta_w(seed):
    g = np.random.default_rng(10 + seed)
    n, d_in, d_out, T = 5, 24, 40, 33
    ranks = g.integers(1, 7, size=n)
    offA, offB, Ap, Bt = make_pools(g, n, d_in, d_out, ranks)
    x = g.standard_normal((T, d_in)); y0 = g.standard_normal((T, d_out))
    ids = g.integers(-1, n, size=T)
    y1 = AP.lora_apply(x, y0, ids, ranks, offA, offB, Ap, Bt, 1.5)
    y2 = AP.lora_apply_dense(x, y0, ids, ranks, offA, offB, Ap, Bt, 1.5)
    np.testing.assert_allclose(y1, y2, atol=1e-12)
    # rows without an adapter are untouched, bit for bit
    np.testing.assert_array_equal(y1[ids < 0], y0[ids < 0])
    # s = 0 leaves y as it is
    np.testing.assert_array_equal(AP.lora_apply(x, y0, ids, ranks, offA, offB, Ap, Bt, 0.0), y0)
    # linear in x
    z = AP.lora_apply(2 * x, 0 * y0, ids, ranks, offA, offB, Ap, Bt, 1.5)
    z1 = AP.lora_apply(x, 0 * y0, ids, ranks, offA, offB, Ap, Bt, 1.5)
    np.testing.assert_allclose(z, 2 * z1, atol=1e-12)
    # permuting tokens permutes the output
    p = g.permutation(T)
    y3 = AP.lora_apply(x[p], y0[p], ids[p], ranks, offA, offB, Ap, Bt, 1.5)
    np.testing.assert_allclose(y3, y1[p], atol=1e-12)


def test_empty_batch():
    y = AP.lora_apply(np.zeros((0, 4)), np.zeros((0, 6)), [], [1], [0], [0], np.ones(4), np.ones(6), 2.0)
    assert y.shape == (0, 6)


def _slice_case(seed):
    g = np.random.default_rng(seed)
    T, n, d_in = 23, 5, 16
    widths = [24, 8, 16]
    slices, y_off = [], 0
    for d_out in widths:
        ranks = g.integers(0, 5, size=n)
        offA = np.concatenate([[0], np.cumsum(ranks * d_in)])
        offB = np.concatenate([[0], np.cumsum(ranks * d_out)])
        slices.append((d_out, y_off, ranks, offA[:-1], offB[:-1], g.standard_normal(int(offA[-1])),
                       g.standard_normal(int(offB[-1]))))
        y_off += d_out + 8            # gaps between slices stay untouched
    ids = g.integers(-1, n, size=T)
    x = g.standard_normal((T, d_in))
    y0 = g.standard_normal((T, y_off))
    return ids, x, y0, slices


@pytest.mark.parametrize("seed", [0, 1])
def test_slices_equal_per_projection_apply(seed):
    # each slice is one projection's side path: the multi-slice definition must equal
    # lora_apply on every slice's columns and leave the gaps between slices alone
    ids, x, y0, slices = _slice_case(seed)
    y = AP.lora_apply_slices(x, y0, ids, slices, 1.5)
    covered = np.zeros(y0.shape[1], dtype=bool)
    for d_out, y_off, ranks, offA, offB, Ap, Bt in slices:
        want = AP.lora_apply(x, y0[:, y_off:y_off + d_out], ids, ranks, offA, offB, Ap, Bt, 1.5)
        np.testing.assert_allclose(y[:, y_off:y_off + d_out], want, rtol=1e-13, atol=1e-13)
        covered[y_off:y_off + d_out] = True
    assert np.array_equal(y[:, ~covered], y0[:, ~covered])


def test_slices_per_adapter_scale():
    # a per-adapter scale scales each token's delta by its own adapter's value only
    ids, x, y0, slices = _slice_case(3)
    n = len(slices[0][2])
    sc = np.arange(1, n + 1, dtype=np.float64)
    y = AP.lora_apply_slices(x, y0, ids, slices, 0.0, adapter_scale=sc)
    for a in range(n):
        one = AP.lora_apply_slices(x, y0, np.where(ids == a, a, -1), slices, 1.0)
        rows = ids == a
        np.testing.assert_allclose(y[rows] - y0[rows], sc[a] * (one[rows] - y0[rows]), rtol=1e-12, atol=1e-12)
    assert np.array_equal(y[ids < 0], y0[ids < 0])


def _sandwich_case(seed, n=4, T=19, d_in=12, d_out=10, r=3):
    g = np.random.default_rng(seed)
    return (g.integers(-1, n, size=T), g.standard_normal((T, d_in)), g.standard_normal((T, d_out)),
            g.standard_normal((r, d_in)), g.standard_normal((r, d_out)))


@pytest.mark.parametrize("diagonal", [True, False])
def test_sigma_sandwich_equals_dense_adapter_matrices(diagonal):
    # brute force: materialise each adapter's dW_a = U Sigma_a V^T and apply it densely
    ids, x, y0, Vt, Ut = _sandwich_case(1)
    g = np.random.default_rng(2)
    sig = g.standard_normal((4, 3)) if diagonal else g.standard_normal((4, 3, 3))
    y = AP.sigma_sandwich_apply(x, y0, ids, Vt, Ut, sig, diagonal, 0.7)
    for t in range(len(ids)):
        a = int(ids[t])
        if a < 0:
            assert np.array_equal(y[t], y0[t])
            continue
        S = np.diag(sig[a]) if diagonal else sig[a]
        dW = Ut.T @ S @ Vt
        np.testing.assert_allclose(y[t], y0[t] + 0.7 * dW @ x[t], rtol=1e-12, atol=1e-12)


def test_sigma_sandwich_identity_sigma_is_a_shared_lora():
    # Sigma_a = I for every adapter: every adapter is the same LoRA (A' = V^T, B'^T = U^T),
    # so the result equals lora_apply with shared factors
    ids, x, y0, Vt, Ut = _sandwich_case(3)
    n, r = 4, 3
    y = AP.sigma_sandwich_apply(x, y0, ids, Vt, Ut, np.tile(np.eye(r), (n, 1, 1)), False, 1.3)
    ranks = np.full(n, r)
    y_ref = AP.lora_apply(x, y0, ids, ranks, np.zeros(n, np.int64), np.zeros(n, np.int64), Vt.ravel(), Ut.ravel(), 1.3)
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)
    # and a diagonal Sigma equals the full form with that diagonal
    d = np.random.default_rng(4).standard_normal((n, r))
    np.testing.assert_allclose(AP.sigma_sandwich_apply(x, y0, ids, Vt, Ut, d, True, 0.5),
                               AP.sigma_sandwich_apply(x, y0, ids, Vt, Ut, np.stack([np.diag(v) for v in d]), False, 0.5),
                               rtol=1e-12, atol=1e-12)
