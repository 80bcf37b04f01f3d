"""Pins of the pool-wide subspace oracle (oracle/pool.py) against closed forms.

LoRASpace (arXiv listing abstract): the minimal subspace of a pool's stacked factors
that keeps 99 % of their energy, by SVD.  Each pin below fixes a property the
mathematics determines without the oracle's own route: planted spectra, duplicated
LoRAs, planted shared bases, the Frobenius energy identity, Eckart-Young for the
projection residual, and the row/column duality of the two stacks.
"""
import math

import numpy as np
import pytest

from oracle import pool as OPL

pytestmark = pytest.mark.filterwarnings("error")


def orthonormal(d, m, g):
    q, _ = np.linalg.qr(g.standard_normal((d, m)))
    return q


def test_equal_energy_orthogonal_pool_needs_ceil_99_percent():
    """Rows mutually orthonormal across the pool, all scaled by c: every singular value
    of the stack equals c, so the smallest k with 100 k >= 99 sum_r is ceil(0.99 sum_r)."""
    g = np.random.default_rng(1)
    ranks = [16, 8, 12, 24]
    d, tot = 200, sum(ranks)
    Q = orthonormal(d, tot, g).T * 3.0                # tot x d, orthogonal rows of norm 3
    As, o = [], 0
    for r in ranks:
        As.append(Q[o:o + r])
        o += r
    res = OPL.pool_subspace(As, "row")
    assert res["k"] == math.ceil(0.99 * tot) == 60
    assert np.allclose(res["sigma"], 3.0, rtol=1e-12)
    assert res["frac"] == 60 / tot
    # at 50 %: exactly half of the equal directions
    assert OPL.pool_subspace(As, "row", 1, 2)["k"] == tot // 2


def test_duplicated_lora_adds_no_direction():
    """N copies of one A: the stack's singular values are sqrt(N) times A's, so the
    pool keeps as many directions as the single LoRA (threshold counted by brute force
    on A A^T's eigenvalues)."""
    g = np.random.default_rng(2)
    r, d, N = 12, 90, 5
    A = np.diag(np.geomspace(1.0, 1e-3, r)) @ orthonormal(d, r, g).T
    lam = np.sort(np.linalg.eigvalsh(A @ A.T))[::-1]   # sigma(A)^2
    k_single = next(k for k in range(1, r + 1) if 100 * lam[:k].sum() >= 99 * lam.sum())
    res = OPL.pool_subspace([A] * N, "row")
    assert res["k"] == k_single
    assert np.allclose(res["sigma"][:r] ** 2, N * lam, rtol=1e-10)
    assert np.all(res["sigma"][r:] <= 1e-12 * res["sigma"][0])


def test_planted_shared_basis_bounds_and_recovers_the_subspace():
    """A_i = C_i Q^T with a shared orthonormal Q (d x m): the stack has rank <= m, so
    k <= m, and at 100 % of the energy the subspace is exactly span(Q)."""
    g = np.random.default_rng(3)
    d, m = 120, 10
    Q = orthonormal(d, m, g)
    As = [g.standard_normal((r, m)) @ Q.T for r in (8, 8, 6, 4)]   # sum r = 26 > m
    res = OPL.pool_subspace(As, "row")
    assert res["k"] <= m
    full = OPL.pool_subspace(As, "row", 1, 1)
    # sigma past m is rounding (~1e-15 relative); 100 % keeps exactly the m real ones
    # unless rounding adds tail energy, which the threshold comparison may count: the
    # first m directions must hold all but rounding of the energy
    assert full["k"] >= m
    P = full["basis"][:, :m]
    assert np.allclose(P @ P.T, Q @ Q.T, atol=1e-10)
    assert res["frac"] == res["k"] / 26


def test_energy_is_the_sum_of_the_factors_frobenius_norms():
    g = np.random.default_rng(4)
    As = [g.standard_normal((r, 64)) for r in (3, 7, 16)]
    Bs = [g.standard_normal((80, r)) for r in (5, 9)]
    assert math.isclose(OPL.pool_subspace(As, "row")["energy"], sum(float(np.sum(a * a)) for a in As), rel_tol=1e-12)
    assert math.isclose(OPL.pool_subspace(Bs, "col")["energy"], sum(float(np.sum(b * b)) for b in Bs), rel_tol=1e-12)


@pytest.mark.parametrize("side", ["row", "col"])
def test_projection_residual_is_the_discarded_energy(side):
    """Eckart-Young for the stack: projecting every factor onto the k leading directions
    leaves exactly sum_{j >= k} sigma_j^2; with k - 1 directions the kept energy falls
    below 99 % (minimality)."""
    g = np.random.default_rng(5)
    spec = np.geomspace(1.0, 1e-2, 40)
    if side == "row":
        F = (np.diag(spec) @ orthonormal(150, 40, g).T)
        F = orthonormal(40, 40, g) @ F                      # mix the rows
        facs = [F[0:16], F[16:24], F[24:40]]
    else:
        F = orthonormal(150, 40, g) @ np.diag(spec) @ orthonormal(40, 40, g).T
        facs = [F[:, 0:16], F[:, 16:24], F[:, 24:40]]
    res = OPL.pool_subspace(facs, side)
    k, s = res["k"], res["sigma"]
    assert np.allclose(s, spec, rtol=1e-10)
    _, resid = OPL.project_pool(facs, res["basis"], side)
    assert math.isclose(resid, float(np.sum(spec[k:] ** 2)), rel_tol=1e-9, abs_tol=1e-15)
    _, resid1 = OPL.project_pool(facs, res["basis"][:, :k - 1], side)
    assert 100 * (res["energy"] - resid1) < 99 * res["energy"] <= 100 * (res["energy"] - resid)


def test_row_and_column_stacks_are_dual():
    """Stacking B_i side by side is stacking B_i^T as rows, transposed: same singular
    values and k, left vectors of one = right vectors of the other (up to sign)."""
    g = np.random.default_rng(6)
    Bs = [g.standard_normal((70, r)) * (1 + i) for i, r in enumerate((4, 6, 5))]
    c = OPL.pool_subspace(Bs, "col")
    rr = OPL.pool_subspace([b.T for b in Bs], "row")
    assert c["k"] == rr["k"]
    assert np.allclose(c["sigma"], rr["sigma"], rtol=1e-12)
    assert np.allclose(np.abs(np.sum(c["basis"] * rr["basis"], axis=0)), 1.0, atol=1e-9)


def test_rank_one_pool_and_full_energy():
    g = np.random.default_rng(7)
    v = orthonormal(50, 1, g).T
    As = [np.array([[2.0]]) @ v, np.array([[-1.0], [0.5]]) @ v]   # every row parallel to v
    res = OPL.pool_subspace(As, "row")
    assert res["k"] == 1 and res["frac"] == 1 / 3
    assert np.allclose(np.abs(res["basis"][:, 0]), np.abs(v[0]), atol=1e-12)
    # generic full-rank stack (sum r <= d) at 100 %: every direction is needed
    As = [g.standard_normal((r, 40)) for r in (6, 9)]
    full = OPL.pool_subspace(As, "row", 1, 1)
    assert full["k"] == 15 and full["frac"] == 1.0


def test_shape_checks():
    with pytest.raises(ValueError):
        OPL.pool_subspace([np.zeros((2, 5)), np.zeros((2, 6))], "row")
    with pytest.raises(ValueError):
        OPL.pool_subspace([np.zeros((5, 2)), np.zeros((6, 2))], "col")
    with pytest.raises(ValueError):
        OPL.pool_subspace([np.zeros((2, 5))], "diag")
