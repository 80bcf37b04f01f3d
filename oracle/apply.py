"""Adapter routing and the multi-LoRA side path, in float64.

Sources
-------
* "Compress then Serve" (academ.us/article/2407.00066), §3: the adapted
  output is (W0 + B A) x; the LoRA term is computed apart from W0 x and added.
* Same page, §11 "Avoiding Batched Matrix Multiplication (BMM)": a batch mixes
  requests for different adapters; the side path is A x, then B (A x).
* Same page, §13.4 "Punica": the steps are buffer = A x with an fp32
  intermediate buffer indexed per token by ``indices``, then y += scale * B buffer.
* Same page, §10 (LoraConfig r=16, lora_alpha=32): the scale s = alpha / r.
* LoRAForge (kongchang.com), "The Bottleneck of Multi-LoRA Serving": adapters
  of different ranks run together in one batch.

Readings:
* Token id -1 means "no adapter": the row of y is left as it is.  An id
  >= n_adapters is an error.
* Routing is a stable sort of tokens by adapter id; segments are runs of
  equal id in ascending adapter order.
* The scale s is the original adapter's alpha / r and is not re-derived from
  the retained rank.
"""
from __future__ import annotations

import numpy as np


def route(ids, n_adapters: int):
    """Stable routing of tokens to adapters.

    Returns (segments int32[n_seg, 3] rows (adapter, start, length),
    perm int32[n_valid]) where perm lists the token indices with id >= 0,
    ordered by (id, token index), and segment s covers perm[start:start+length].
    """
    ids = np.asarray(ids, dtype=np.int64)
    if np.any(ids < -1) or np.any(ids >= n_adapters):
        raise ValueError("adapter id out of range")
    valid = np.nonzero(ids >= 0)[0]
    perm = valid[np.argsort(ids[valid], kind="stable")]
    segs = []
    start = 0
    while start < len(perm):
        a = ids[perm[start]]
        end = start
        while end < len(perm) and ids[perm[end]] == a:
            end += 1
        segs.append((int(a), start, end - start))
        start = end
    return np.array(segs, dtype=np.int32).reshape(-1, 3), perm.astype(np.int32)


def adapter_factors(a: int, ranks, off_A, off_Bt, A_pool, Bt_pool, d_in: int, d_out: int):
    """(A' k x d_in, B'^T k x d_out) of adapter a from packed pools, as float64."""
    k = int(ranks[a])
    oa, ob = int(off_A[a]), int(off_Bt[a])
    Ap = np.asarray(A_pool[oa:oa + k * d_in], dtype=np.float64).reshape(k, d_in)
    Bt = np.asarray(Bt_pool[ob:ob + k * d_out], dtype=np.float64).reshape(k, d_out)
    return Ap, Bt


def lora_apply(x, y0, ids, ranks, off_A, off_Bt, A_pool, Bt_pool, scale: float):
    """y = y0 + s * B'_a (A'_a x_t) for every token t with adapter a = ids[t] >= 0.

    x: T x d_in, y0: T x d_out (any float dtype, taken exactly), pools: flat
    arrays holding each adapter's A' (k x d_in) and B'^T (k x d_out) row-major
    at the given element offsets.  Returns y in float64 (no output rounding).
    """
    x = np.asarray(x, dtype=np.float64)
    y = np.array(y0, dtype=np.float64, copy=True)
    T, d_in = x.shape
    d_out = y.shape[1]
    segs, perm = route(ids, len(ranks))
    for a, start, length in segs:
        rows = perm[start:start + length]
        Ap, Bt = adapter_factors(a, ranks, off_A, off_Bt, A_pool, Bt_pool, d_in, d_out)
        t = x[rows] @ Ap.T              # intermediate, one value per retained direction
        y[rows] += scale * (t @ Bt)
    return y


def lora_apply_dense(x, y0, ids, ranks, off_A, off_Bt, A_pool, Bt_pool, scale: float):
    """Brute force: materialise Delta W'_a = B'_a A'_a and multiply each token by it."""
    x = np.asarray(x, dtype=np.float64)
    y = np.array(y0, dtype=np.float64, copy=True)
    T, d_in = x.shape
    d_out = y.shape[1]
    ids = np.asarray(ids)
    for t in range(T):
        a = int(ids[t])
        if a < 0:
            continue
        Ap, Bt = adapter_factors(a, ranks, off_A, off_Bt, A_pool, Bt_pool, d_in, d_out)
        y[t] = y[t] + scale * ((Bt.T @ Ap) @ x[t])
    return y


def lora_apply_slices(x, y0, ids, slices, scale: float, adapter_scale=None):
    """Side path of several output slices that share x ("Compress then Serve" §13.4:
    the LoRA buffer comes from x per token and is added to each projection's output).

    slices: list of (d_out, y_offset, ranks, off_A, off_Bt, A_pool, Bt_pool); y0 is
    T x y_ld and slice s occupies columns y_offset .. y_offset + d_out.  For every
    token t with adapter a = ids[t] >= 0 and every slice:
        y[t, slice] += scale_a * B'_{s,a} (A'_{s,a} x_t),
    scale_a = adapter_scale[a] when given, else scale.  Columns outside the slices
    keep y0.  Returns y in float64.
    """
    x = np.asarray(x, dtype=np.float64)
    y = np.array(y0, dtype=np.float64, copy=True)
    ids = np.asarray(ids)
    n_adapters = len(slices[0][2])
    if np.any(ids < -1) or np.any(ids >= n_adapters):
        raise ValueError("adapter id out of range")
    d_in = x.shape[1]
    for t in range(x.shape[0]):
        a = int(ids[t])
        if a < 0:
            continue
        sa = float(adapter_scale[a]) if adapter_scale is not None else scale
        for d_out, y_off, ranks, off_A, off_Bt, A_pool, Bt_pool in slices:
            Ap, Bt = adapter_factors(a, ranks, off_A, off_Bt, A_pool, Bt_pool, d_in, d_out)
            y[t, y_off:y_off + d_out] += sa * (Bt.T @ (Ap @ x[t]))
    return y


def sigma_sandwich_apply(x, y0, ids, Vt, Ut, sigma, diagonal: bool, scale: float):
    """Serving of jointly compressed adapters ("Compress then Serve" §3.1, §11):
    B_a A_a ~ U Sigma_a V^T with U, V shared by all adapters and a small Sigma_a each;
    for every token t with a = ids[t] >= 0,  y_t += scale * U (Sigma_a (V^T x_t)).

    Vt = V^T (rank x d_in), Ut = U^T (rank x d_out); sigma: n_adapters x rank
    (diagonal Sigma_a) or n_adapters x rank x rank (full).  Returns y in float64.
    """
    x = np.asarray(x, dtype=np.float64)
    y = np.array(y0, dtype=np.float64, copy=True)
    Vt = np.asarray(Vt, dtype=np.float64); Ut = np.asarray(Ut, dtype=np.float64)
    sig = np.asarray(sigma, dtype=np.float64)
    ids = np.asarray(ids)
    n = sig.shape[0]
    if np.any(ids < -1) or np.any(ids >= n):
        raise ValueError("adapter id out of range")
    for t in range(x.shape[0]):
        a = int(ids[t])
        if a < 0:
            continue
        z = Vt @ x[t]                                   # V^T x
        w = sig[a] * z if diagonal else sig[a] @ z      # Sigma_a (V^T x)
        y[t] += scale * (Ut.T @ w)                      # U (...)
    return y
