"""Pins for oracle.factor against closed forms, independent routines and hand cases.

Nothing here re-calls the routine under test to produce its own expected
value: QR is pinned by hand cases, the Gram identity and classical
Gram-Schmidt; the spectrum by planted singular values, a 2x2 closed form and
the eigenvalues of Delta W^T Delta W; truncation by Eckart-Young.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import factor as F
from tests.conftest import GOLDEN

GOLD = json.load(open(os.path.join(GOLDEN, "small_factors.json")))


def rng(seed):
    return np.random.default_rng(seed)


def orthonormal(m, n, seed):
    # Gram-Schmidt of a Gaussian, written out (independent of numpy's QR)
    G = rng(seed).standard_normal((m, n))
    Q = np.zeros((m, n))
    for j in range(n):
        v = G[:, j].copy()
        for _ in range(2):
            v -= Q[:, :j] @ (Q[:, :j].T @ v)
        Q[:, j] = v / np.linalg.norm(v)
    return Q


@pytest.mark.parametrize("case", GOLD["qr"])
def test_qr_hand_cases(case):
    R = F.qr_r(np.array(case["X"], dtype=float))
    np.testing.assert_allclose(R, np.array(case["R"], dtype=float), atol=1e-14)


def test_qr_gram_schmidt_and_invariants():
    X = rng(1).standard_normal((200, 12)) * np.logspace(0, -3, 12)
    R = F.qr_r(X)
    assert np.allclose(R, np.triu(R))
    assert np.all(np.diag(R) >= 0)
    # Gram identity R^T R = X^T X
    np.testing.assert_allclose(R.T @ R, X.T @ X, rtol=1e-12, atol=1e-14 * np.abs(X.T @ X).max())
    # classical Gram-Schmidt with re-orthogonalisation gives the same R
    m, n = X.shape
    Q = np.zeros((m, n)); Rg = np.zeros((n, n))
    for j in range(n):
        v = X[:, j].copy()
        c = Q[:, :j].T @ v; v -= Q[:, :j] @ c
        c2 = Q[:, :j].T @ v; v -= Q[:, :j] @ c2
        Rg[:j, j] = c + c2
        Rg[j, j] = np.linalg.norm(v)
        Q[:, j] = v / Rg[j, j]
    np.testing.assert_allclose(R, Rg, rtol=1e-9, atol=1e-12)
    Qo = F.qr_q(X)
    np.testing.assert_allclose(Qo.T @ Qo, np.eye(n), atol=1e-13)
    np.testing.assert_allclose(Qo @ R, X, atol=1e-13)


def test_planted_spectrum_both_routes():
    d_out, d_in, r = 96, 80, 8
    sig = np.array([5.0, 3.0, 2.0, 1.5, 1.0, 0.5, 0.25, 0.125])
    Q1 = orthonormal(d_out, r, 2); Q2 = orthonormal(d_in, r, 3)
    B = Q1 * sig          # B = Q1 diag(sigma)
    A = Q2.T              # A = Q2^T  ->  Delta W = Q1 diag(sigma) Q2^T
    s_d, U_d, Vt_d = F.spectrum_dense(B, A)
    s_f, U_M, R_B, R_A = F.spectrum_factor(B, A)
    np.testing.assert_allclose(s_d, sig, rtol=1e-13)
    np.testing.assert_allclose(s_f, sig, rtol=1e-13)
    # left singular vectors span the planted directions (|U^T Q1| = I)
    np.testing.assert_allclose(np.abs(U_d.T @ Q1), np.eye(r), atol=1e-12)


def test_two_by_two_closed_form():
    # for M = [[a, b], [0, d]]: s1^2 + s2^2 = a^2+b^2+d^2, s1 s2 = |a d|
    a, b, d = 3.0, 4.0, 2.0
    B = np.array([[a, b], [0.0, d]]); A = np.eye(2)
    s, *_ = F.spectrum_dense(B, A)
    tot = a * a + b * b + d * d; prod = abs(a * d)
    s1 = math.sqrt((tot + math.sqrt(tot * tot - 4 * prod * prod)) / 2)
    s2 = prod / s1
    np.testing.assert_allclose(s, [s1, s2], rtol=1e-14)


def test_dense_spectrum_matches_gram_eigenvalues():
    g = rng(4)
    B = g.standard_normal((40, 6)); A = g.standard_normal((6, 30))
    s, U, Vt = F.spectrum_dense(B, A)
    W = B @ A
    ev = np.sort(np.linalg.eigvalsh(W.T @ W))[::-1][:6]
    np.testing.assert_allclose(s * s, ev, rtol=1e-10)
    # U columns are eigenvectors of W W^T with eigenvalue s^2
    np.testing.assert_allclose((W @ W.T) @ U, U * (s * s), atol=1e-9 * s[0] ** 2)


def test_factor_route_matches_definition_route():
    g = rng(5)
    d_out, d_in, r = 150, 110, 10
    B = (g.standard_normal((d_out, r)) * (1.0 / np.arange(1, r + 1))).astype(np.float32)
    A = (g.standard_normal((r, d_in)) / math.sqrt(d_in)).astype(np.float32)
    s_d, *_ = F.spectrum_dense(B, A)
    s_f, *_ = F.spectrum_factor(B, A)
    np.testing.assert_allclose(s_f, s_d, rtol=0, atol=1e-12 * s_d[0])


@pytest.mark.parametrize("case", GOLD["truncation"])
def test_truncation_error_hand(case):
    assert F.truncation_error(case["sigma"], case["k"]) == pytest.approx(case["err"], abs=1e-15)


@pytest.mark.parametrize("route", ["dense", "factor"])
def test_eckart_young_and_export(route):
    g = rng(6)
    d_out, d_in, r = 120, 90, 8
    B = g.standard_normal((d_out, r)) * (1.0 / np.arange(1, r + 1))
    A = g.standard_normal((r, d_in)) / math.sqrt(d_in)
    s, *_ = F.spectrum_dense(B, A)
    exp = F.export_dense if route == "dense" else F.export_factor
    for k in range(0, r + 1):
        Bt, Ap = exp(B, A, k)
        assert Bt.shape == (k, d_out) and Ap.shape == (k, d_in)
        if k:
            np.testing.assert_allclose(Bt @ Bt.T, np.eye(k), atol=1e-12)  # B' orthonormal
        err = F.dense_error(B, A, Bt, Ap)
        assert err == pytest.approx(F.truncation_error(s, k), abs=1e-12)
        assert F.factor_error(B, A, Bt, Ap) == pytest.approx(err, abs=1e-7)
    Bt, Ap = exp(B, A, r)
    assert F.dense_error(B, A, Bt, Ap) < 1e-12            # exact at k = r


def test_export_routes_agree_on_product():
    g = rng(7)
    B = g.standard_normal((64, 6)); A = g.standard_normal((6, 48))
    for k in (1, 3, 6):
        Bt1, Ap1 = F.export_dense(B, A, k)
        Bt2, Ap2 = F.export_factor(B, A, k)
        np.testing.assert_allclose(Bt1.T @ Ap1, Bt2.T @ Ap2, atol=1e-11)


def test_factor_error_detects_wrong_factors():
    g = rng(8)
    B = g.standard_normal((50, 4)); A = g.standard_normal((4, 40))
    Bt, Ap = F.export_dense(B, A, 4)
    Ap_bad = Ap.copy(); Ap_bad[0] *= -1
    assert F.factor_error(B, A, Bt, Ap_bad) == pytest.approx(F.dense_error(B, A, Bt, Ap_bad), rel=1e-9)
    assert F.factor_error(B, A, Bt, Ap_bad) > 0.1


def test_zero_module():
    B = np.zeros((20, 3)); A = np.zeros((3, 10))
    assert F.truncation_error(np.zeros(3), 1) == 0.0
    R = F.qr_r(B)
    assert np.all(R == 0)
