"""GPU parity of the pool-wide subspace of stacked row factors (LoRASpace, the arXiv
listing abstract) against the fp64 oracle on the same fp32 bytes.

The stack of a pool's A_i goes through lf_tsqr_batched as one module with an identity
partner factor, then the energy-fraction policy picks k.  Each pool plants a shared
basis with a graded spectrum plus small independent noise, and the test asserts that
the 99 % (or 90 %) threshold is not within 1e-3 of a tie, so k is fixed in fp32 as well
as fp64.  Tolerances: k exact; sigma within 2e-5 sigma_1 (the factor path's bound).
"""
import numpy as np
import pytest
import torch

from oracle import allocate as OA
from oracle import pool as OPL
from post_hoc_rank_b200 import api, build
from post_hoc_rank_b200 import loraforge as lf

pytestmark = pytest.mark.gpu

SIG_TOL = 2e-5


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available()


def make_pool(ranks, d_in, m, key):
    g = np.random.default_rng(key)
    Q, _ = np.linalg.qr(g.standard_normal((d_in, m)))
    spec = np.geomspace(1.0, 0.05, m)
    flat, offs, o = [], [], 0
    for r in ranks:
        C = g.standard_normal((r, m)) * spec
        A = C @ Q.T + 1e-3 * g.standard_normal((r, d_in)) / np.sqrt(d_in)
        flat.append(A.astype(np.float32).reshape(-1))
        offs.append(o)
        o += r * d_in
    return np.concatenate(flat), offs


@pytest.mark.parametrize("ranks,d_in,m,num,den", [
    ([16, 16, 16, 16], 4096, 20, 99, 100),
    ([16, 8, 12, 4], 3584, 20, 99, 100),
    ([32, 32], 1024, 40, 9, 10),
    ([13, 7, 1], 333, 12, 99, 100),
])
def test_pool_subspace_matches_oracle(ranks, d_in, m, num, den):
    flat, offs = make_pool(ranks, d_in, m, (len(ranks), d_in))
    As = [flat[o:o + r * d_in].astype(np.float64).reshape(r, d_in) for o, r in zip(offs, ranks)]
    want = OPL.pool_subspace(As, "row", num, den)
    _, gap = OA.energy_fraction_rank(want["sigma"], len(want["sigma"]), num, den, 1)
    assert gap > 1e-3
    k, sig, _ = api.pool_subspace_rows(torch.from_numpy(flat).cuda(), offs, ranks, d_in, num, den)
    assert lf.lf_get_device_status() == 0
    assert k == want["k"]
    s = sig.cpu().numpy()
    assert np.max(np.abs(s - want["sigma"])) <= SIG_TOL * want["sigma"][0]


def make_factors(ranks, d, m, key, side, dup=None):
    """Pool of LoRA factors around a planted shared basis (m directions, graded spectrum)
    plus small independent noise; side "row": A_i (r_i x d), "col": B_i (d x r_i), stored
    back to back (row-major) in one fp32 buffer.  dup = (i, j): factor j repeats factor i
    (a rank-deficient stack)."""
    g = np.random.default_rng(key)
    Q, _ = np.linalg.qr(g.standard_normal((d, m)))
    spec = np.geomspace(1.0, 0.05, m)
    rows = []
    for r in ranks:
        C = g.standard_normal((r, m)) * spec
        rows.append((C @ Q.T + 1e-3 * g.standard_normal((r, d)) / np.sqrt(d)).astype(np.float32))
    if dup is not None:
        rows[dup[1]] = rows[dup[0]].copy()
    fs = [f if side == "row" else np.ascontiguousarray(f.T) for f in rows]
    offs = np.concatenate([[0], np.cumsum([f.size for f in fs])[:-1]]).astype(np.int64)
    flat = np.concatenate([f.reshape(-1) for f in fs])
    return flat, offs, [f.astype(np.float64) for f in fs]


@pytest.mark.parametrize("side", ["row", "col"])
@pytest.mark.parametrize("ranks,d,m,dup", [
    ([16] * 8, 4096, 40, None),        # summed rank 128
    ([16] * 17, 4096, 100, None),      # a 17-LoRA pool, summed rank 272
    ([32] * 16, 14336, 200, None),     # summed rank 512 (the limit), ffn-wide factors
    ([13, 7, 1, 40, 3], 1000, 30, None),
    ([16] * 4, 2048, 24, (0, 2)),      # one LoRA repeated: a rank-deficient stack
])
def test_pool_subspace_on_the_gpu_matches_oracle(side, ranks, d, m, dup):
    """lf_pool_subspace against the fp64 oracle (numpy SVD of the stack, the energy
    fraction rule, projection of every factor on the basis): k exact, sigma within
    2e-5 sigma_1, the k-dimensional subspace (projector distance), an orthonormal basis,
    the projection residual, and every factor rebuilt from the GPU's coefficients."""
    flat, offs, fs = make_factors(ranks, d, m, (len(ranks), d, m), side, dup)
    want = OPL.pool_subspace(fs, side, 99, 100)
    _, gap = OA.energy_fraction_rank(want["sigma"], len(want["sigma"]), 99, 100, 1)
    # not a tie: the GPU's energies come from the exact fp64 Gram of the same fp32 bytes
    # (about 1e-13 of the total), far inside a relative gap of 1e-8
    assert gap > 1e-8
    out = api.pool_subspace(torch.from_numpy(flat).cuda(), offs, ranks, d, side, 99, 100)
    assert lf.lf_get_device_status() == 0
    k = int(out.k.item())
    assert k == want["k"]
    s = out.sigma.cpu().numpy()
    assert np.max(np.abs(s - want["sigma"])) <= SIG_TOL * want["sigma"][0]
    P = out.basis.double().cpu().numpy()[:k].T          # d x k
    Po = want["basis"]
    assert np.abs(P.T @ P - np.eye(k)).max() <= 1e-5
    # distance of the two projectors onto the k-dimensional subspaces
    dist = np.sqrt(max(2.0 * k - 2.0 * np.sum((P.T @ Po) ** 2), 0.0))
    assert dist <= 1e-3, dist
    _, resid_o = OPL.project_pool(fs, Po, side)
    energy = want["energy"]
    assert abs(float(out.resid.item()) - resid_o) <= 1e-5 * energy
    # every factor from the GPU's coefficients and basis: the same residual
    C = out.coef.double().cpu().numpy()[:, :k]
    resid_g, a0 = 0.0, 0
    for f, r in zip(fs, ranks):
        rec = C[a0:a0 + r] @ P.T if side == "row" else P @ C[a0:a0 + r].T
        resid_g += float(np.sum((f - rec) ** 2))
        a0 += r
    assert abs(resid_g - resid_o) <= 1e-5 * energy


def test_pool_subspace_host_checks():
    L = lf.lib()
    rk = np.array([300, 300], np.int32); of = np.array([0, 300 * 4096], np.int64)
    assert L.lf_pool_workspace_size(0, 2, rk.ctypes.data, of.ctypes.data, 4096) == 0   # R > 512
    rk1 = np.array([16], np.int32); of1 = np.array([0], np.int64)
    assert L.lf_pool_workspace_size(2, 1, rk1.ctypes.data, of1.ctypes.data, 64) == 0   # bad side
    assert L.lf_pool_workspace_size(0, 1, rk1.ctypes.data, of1.ctypes.data, 8) == 0    # R > d
    assert L.lf_pool_workspace_size(1, 1, rk1.ctypes.data, of1.ctypes.data, 64) > 0
