"""Pins for the JD-Full eigenvalue-iteration oracle (oracle/jd.py).

"Compress then Serve" (academ.us/article/2407.00066), §3.1 eq. 1 and Appendix 8.1
(case 1, eqs. 6-7) and 8.2.  Each test checks the oracle against something other
than itself: a second orthogonalisation algorithm, Eckart-Young on a planted
spectrum, an exactly shared basis, the dense d x d operators of Appendix 8.1,
library eigendecompositions of those operators, and the §6 normalisation.
"""
import numpy as np
import pytest

from oracle import jd as OJ


def rng(seed):
    return np.random.default_rng(seed)


def orthonormal(g, m, n):
    q, _ = np.linalg.qr(g.standard_normal((m, n)))
    return q


def mgs(X):
    """Modified Gram-Schmidt: the Q with positive diagonal R, column by column."""
    X = np.array(X, dtype=np.float64)
    m, n = X.shape
    Q = np.zeros_like(X)
    for j in range(n):
        v = X[:, j].copy()
        for i in range(j):
            v -= (Q[:, i] @ v) * Q[:, i]
        Q[:, j] = v / np.linalg.norm(v)
    return Q


def collection(g, n, d_out, d_in, ranks):
    Bs = [g.standard_normal((d_out, r)) / np.sqrt(d_out) for r in ranks[:n]]
    As = [g.standard_normal((r, d_in)) / np.sqrt(d_in) for r in ranks[:n]]
    return Bs, As


def test_orthogonalize_is_the_unique_qr():
    X = rng(1).standard_normal((40, 7))
    Q, R = OJ.orthogonalize(X)
    assert np.allclose(Q.T @ Q, np.eye(7), atol=1e-13)
    assert np.allclose(Q @ R, X, atol=1e-12)
    assert np.allclose(np.tril(R, -1), 0.0) and (np.diag(R) > 0).all()
    assert np.allclose(Q, mgs(X), atol=1e-10)


def test_step_matches_dense_operators():
    """U_0 = M U and V_0 = N V with M, N formed densely (Appendix 8.1)."""
    g = rng(2)
    Bs, As = collection(g, 3, 12, 10, [2, 4, 3])
    U = g.standard_normal((12, 3))
    V = g.standard_normal((10, 3))
    w = [0.5, 2.0, 1.5]
    dW = [B @ A for B, A in zip(Bs, As)]
    M = sum(wi * D @ V @ V.T @ D.T for wi, D in zip(w, dW))
    N = sum(wi * D.T @ U @ U.T @ D for wi, D in zip(w, dW))
    Un, Vn, U0, V0 = OJ.jd_step(Bs, As, U, V, w)
    assert np.allclose(U0, M @ U, rtol=1e-12, atol=1e-14)
    assert np.allclose(V0, N @ V, rtol=1e-12, atol=1e-14)
    assert np.allclose(Un, mgs(M @ U), atol=1e-10)
    assert np.allclose(Vn, mgs(N @ V), atol=1e-10)


def test_sigma_and_residual_match_dense_definitions():
    g = rng(3)
    Bs, As = collection(g, 4, 16, 14, [3, 1, 4, 2])
    U = orthonormal(g, 16, 3)
    V = orthonormal(g, 14, 3)
    S = OJ.sigma_star(Bs, As, U, V)
    for B, A, Si in zip(Bs, As, S):
        assert np.allclose(Si, U.T @ (B @ A) @ V, atol=1e-14)
    S2 = [Si + 0.1 * g.standard_normal(Si.shape) for Si in S]   # any Sigma, any U, V
    U2, V2 = g.standard_normal((16, 3)), g.standard_normal((14, 3))
    res, tot = OJ.jd_residual(Bs, As, U2, V2, S2)
    dense = sum(np.linalg.norm(B @ A - U2 @ Si @ V2.T) ** 2 for B, A, Si in zip(Bs, As, S2))
    assert res == pytest.approx(dense, rel=1e-11)
    assert tot == pytest.approx(sum(np.linalg.norm(B @ A) ** 2 for B, A in zip(Bs, As)), rel=1e-12)
    # eq. 7: with orthonormal bases and Sigma* the retained energy is total - residual
    res_star, _ = OJ.jd_residual(Bs, As, U, V, S)
    assert tot - res_star == pytest.approx(sum(np.linalg.norm(Si) ** 2 for Si in S), rel=1e-11)


def test_single_lora_reaches_eckart_young():
    """n = 1: JD is the truncated SVD (Appendix 8.1), so the residual is the sum of
    the discarded sigma^2 of a planted spectrum and Sigma has the kept sigma."""
    g = rng(4)
    d_out, d_in, r, rt = 30, 24, 6, 3
    sig = np.array([5.0, 3.0, 2.0, 0.5, 0.3, 0.1])
    B = orthonormal(g, d_out, r) * sig[None, :]
    A = orthonormal(g, d_in, r).T
    U, V, S = OJ.jd_full([B], [A], g.standard_normal((d_out, rt)), g.standard_normal((d_in, rt)), 60)
    res, tot = OJ.jd_residual([B], [A], U, V, S)
    assert tot == pytest.approx(float((sig ** 2).sum()), rel=1e-12)
    assert res == pytest.approx(float((sig[rt:] ** 2).sum()), rel=1e-9)
    assert np.allclose(np.linalg.svd(S[0], compute_uv=False), sig[:rt], rtol=1e-9)
    assert np.allclose(U.T @ U, np.eye(rt), atol=1e-13)


def test_shared_basis_is_recovered():
    """B_i A_i = U* S_i V*^T exactly: the optimum of eq. 1 is zero and the
    iteration finds span(U*), span(V*)."""
    g = rng(5)
    d_out, d_in, rt, n = 40, 36, 4, 5
    Us, Vs = orthonormal(g, d_out, rt), orthonormal(g, d_in, rt)
    Ss = [g.standard_normal((rt, rt)) for _ in range(n)]
    Bs = [Us @ S for S in Ss]
    As = [Vs.T.copy() for _ in range(n)]
    U, V, S = OJ.jd_full(Bs, As, g.standard_normal((d_out, rt)), g.standard_normal((d_in, rt)), 40)
    res, tot = OJ.jd_residual(Bs, As, U, V, S)
    assert abs(res) <= 1e-13 * tot   # the factor-space identity cancels to ~u * total
    assert np.allclose(U @ U.T, Us @ Us.T, atol=1e-10)
    assert np.allclose(V @ V.T, Vs @ Vs.T, atol=1e-10)
    for Si, B, A in zip(S, Bs, As):
        assert np.allclose(U @ Si @ V.T, B @ A, atol=1e-10)


def test_fixed_point_is_the_top_eigenspace():
    """At convergence U holds the top-r~ eigenvectors of M(V) and V those of N(U)
    (Appendix 8.1, case 1), checked with a library symmetric eigensolver."""
    g = rng(6)
    d_out, d_in, rt = 20, 18, 3
    Us, Vs = orthonormal(g, d_out, rt), orthonormal(g, d_in, rt)
    Bs, As = [], []
    for i in range(4):   # a dominant shared part plus small individual parts
        Bs.append(np.hstack([Us @ (np.diag([4.0, 3.0, 2.0]) + 0.3 * g.standard_normal((rt, rt))),
                             0.2 * g.standard_normal((d_out, 2))]))
        As.append(np.vstack([Vs.T, g.standard_normal((2, d_in))]))
    U, V, _ = OJ.jd_full(Bs, As, g.standard_normal((d_out, rt)), g.standard_normal((d_in, rt)), 300)
    dW = [B @ A for B, A in zip(Bs, As)]
    M = sum(D @ V @ V.T @ D.T for D in dW)
    N = sum(D.T @ U @ U.T @ D for D in dW)
    eu = np.linalg.eigh(M)[1][:, -rt:]
    ev = np.linalg.eigh(N)[1][:, -rt:]
    assert np.allclose(U @ U.T, eu @ eu.T, atol=1e-8)
    assert np.allclose(V @ V.T, ev @ ev.T, atol=1e-8)


def test_weights_are_the_unit_norm_normalisation():
    """§6: JD on unit-norm products with the norms restored equals JD with
    w_i = 1 / ||B_i A_i||_F^2 and Sigma_i = U^T B_i A_i V."""
    g = rng(7)
    Bs, As = collection(g, 3, 15, 13, [3, 2, 4])
    Bs[1] = Bs[1] * 10.0
    nrm = [np.linalg.norm(B @ A) for B, A in zip(Bs, As)]
    U0, V0 = g.standard_normal((15, 3)), g.standard_normal((13, 3))
    Uw, Vw, Sw = OJ.jd_full(Bs, As, U0, V0, 7, weights=[1.0 / c ** 2 for c in nrm])
    Un, Vn, Sn = OJ.jd_full([B / c for B, c in zip(Bs, nrm)], As, U0, V0, 7)
    assert np.allclose(Uw, Un, atol=1e-10) and np.allclose(Vw, Vn, atol=1e-10)
    for a, b, c in zip(Sw, Sn, nrm):
        assert np.allclose(a, c * b, atol=1e-10)
    # without the weights the large adapter dominates: a different answer
    Uu, _, _ = OJ.jd_full(Bs, As, U0, V0, 7)
    assert not np.allclose(Uu, Uw, atol=1e-3)


def test_zero_iterations_return_the_start():
    g = rng(8)
    Bs, As = collection(g, 2, 9, 8, [2, 2])
    U0, V0 = g.standard_normal((9, 2)), g.standard_normal((8, 2))
    U, V, S = OJ.jd_full(Bs, As, U0, V0, 0)
    assert np.array_equal(U, U0) and np.array_equal(V, V0)
    assert np.allclose(S[0], U0.T @ Bs[0] @ As[0] @ V0)
