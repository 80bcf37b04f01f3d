"""Joint diagonalization of a LoRA collection (JD-Full) by eigenvalue iteration, fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA path never
imports this module.

Sources
-------
* "Compress then Serve" (academ.us/article/2407.00066), §3.1 "Joint
  Diagonalization", eq. 1: the n LoRA products B_i A_i of one module position are
  approximated as U Sigma_i V^T with U, V shared by all n and one r~ x r~ matrix
  Sigma_i per LoRA; JD-Full keeps U, V with orthonormal columns and Sigma_i full.
* Same page, Appendix 8.1, case 1: for fixed U, V the optimal Sigma_i is
  U^T B_i A_i V (eq. 6), and U, V maximise sum_i ||U^T B_i A_i V||_F^2 (eq. 7).
* Same page, Appendix 8.2 "Additional Eigenvalue Iteration Algorithm": both
  bases are updated from the previous iterate,
      U_0 <- sum_i B_i (A_i V) (V^T A_i^T) (B_i^T U)
      V_0 <- sum_i A_i^T (B_i^T U) (U^T B_i) (A_i V)
      U <- orthogonalize(U_0),  V <- orthogonalize(V_0),
  with orthogonalize the Q factor of the reduced QR, and the products taken in
  that order so no d x d matrix is ever formed.
* Same page, §6 (experimental setup): each LoRA is scaled to unit Frobenius
  norm before JD and its norm is restored afterwards.

Readings (the pages leave these open)
-------------------------------------
* U^(0), V^(0) are inputs, used as given by the first update (they need not be
  orthonormal; the first orthogonalize makes them so).  The pages draw random
  starting bases; the tests pass seeded Gaussian matrices.
* orthogonalize(X) is the Q of X = Q R with diag(R) > 0, which makes it unique
  for a full-column-rank X.
* The normalisation of §6 enters only as a weight: scaling B_i A_i by c_i
  multiplies its terms of U_0 and V_0 by c_i^2 and its Sigma_i by c_i, so JD on
  the normalised collection with the norms restored afterwards equals JD with
  weights w_i = 1 / ||B_i A_i||_F^2 in both sums and Sigma_i = U^T B_i A_i V.
  ``weights=None`` means w_i = 1.
* After the last iteration Sigma_i is eq. 6 at the final U, V.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def orthogonalize(X):
    """Q of the reduced QR X = Q R with diag(R) > 0 (Appendix 8.2's orthogonalize).

    Returns (Q, R).  A library Householder QR followed by the sign choice that
    makes the factorisation unique.
    """
    X = np.asarray(X, dtype=F64)
    Q, R = np.linalg.qr(X, mode="reduced")
    s = np.where(np.diag(R) < 0, -1.0, 1.0)
    return Q * s[None, :], R * s[:, None]


def jd_step(Bs, As, U, V, weights=None):
    """One eigenvalue-iteration step (Appendix 8.2): returns (U_new, V_new, U_0, V_0).

    Bs[i] is d_out x r_i, As[i] is r_i x d_in, U is d_out x r~, V is d_in x r~.
    """
    U = np.asarray(U, dtype=F64)
    V = np.asarray(V, dtype=F64)
    U0 = np.zeros_like(U)
    V0 = np.zeros_like(V)
    for i, (B, A) in enumerate(zip(Bs, As)):
        B = np.asarray(B, dtype=F64)
        A = np.asarray(A, dtype=F64)
        w = 1.0 if weights is None else float(weights[i])
        AV = A @ V            # r_i x r~
        BtU = B.T @ U         # r_i x r~
        U0 += w * (B @ (AV @ (AV.T @ BtU)))
        V0 += w * (A.T @ (BtU @ (BtU.T @ AV)))
    return orthogonalize(U0)[0], orthogonalize(V0)[0], U0, V0


def sigma_star(Bs, As, U, V):
    """Sigma_i = U^T B_i A_i V for every i (Appendix 8.1, eq. 6), as (B_i^T U)^T (A_i V)."""
    U = np.asarray(U, dtype=F64)
    V = np.asarray(V, dtype=F64)
    return [(np.asarray(B, dtype=F64).T @ U).T @ (np.asarray(A, dtype=F64) @ V) for B, A in zip(Bs, As)]


def jd_full(Bs, As, U_init, V_init, iters, weights=None):
    """JD-Full by `iters` eigenvalue-iteration steps from (U_init, V_init).

    Returns (U, V, Sigmas) with Sigmas[i] = U^T B_i A_i V at the final U, V.
    With iters = 0 the bases are returned as given.
    """
    U = np.asarray(U_init, dtype=F64)
    V = np.asarray(V_init, dtype=F64)
    for _ in range(iters):
        U, V, _, _ = jd_step(Bs, As, U, V, weights)
    return U, V, sigma_star(Bs, As, U, V)


def jd_residual(Bs, As, U, V, Sigmas):
    """sum_i ||B_i A_i - U Sigma_i V^T||_F^2 in factor space (eq. 1's objective).

    ||X - Y||^2 = ||X||^2 - 2 <X, Y> + ||Y||^2 with X = B A and Y = U S V^T:
    ||B A||^2 = tr((B^T B)(A A^T)), <B A, U S V^T> = tr(S^T (U^T B)(A V)) and
    ||U S V^T||^2 = tr(S^T (U^T U) S (V^T V)); every product is r x r sized.
    Returns (residual, total) with total = sum_i ||B_i A_i||_F^2.
    """
    U = np.asarray(U, dtype=F64)
    V = np.asarray(V, dtype=F64)
    UtU, VtV = U.T @ U, V.T @ V
    res = tot = 0.0
    for B, A, S in zip(Bs, As, Sigmas):
        B = np.asarray(B, dtype=F64)
        A = np.asarray(A, dtype=F64)
        S = np.asarray(S, dtype=F64)
        nx = float(np.trace((B.T @ B) @ (A @ A.T)))
        cross = float(np.trace(S.T @ ((U.T @ B) @ (A @ V))))
        ny = float(np.trace(S.T @ UtU @ S @ VtV))
        res += nx - 2.0 * cross + ny
        tot += nx
    return res, tot
