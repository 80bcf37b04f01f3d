"""Spectrum, truncation and export of one LoRA module, in float64.

Sources
-------
* "Compress then Serve" (academ.us/article/2407.00066), §3 "Rank-Based LoRA
  Compression": a module's update is Delta W = B A with B d_B x r, A r x d_A,
  and the adapted output is (W0 + B A) x.
* Same page, §4 "Theoretical Analysis", eq. 4: per-module truncated SVD
  SVD_r(B_i A_i) = U_i Sigma_i V_i^T; by Eckart-Young it is the best rank-r
  approximation, and Sigma_i V_i^T is kept as one matrix.
* LoRAForge (kongchang.com), section "FlashTSQR: An Accelerator for Batched
  Factor Construction" and the glossary paragraph before it: TSQR factors a
  tall-skinny matrix by local QR of row blocks followed by merging.  Its
  result is the R factor of the thin QR, which is unique once diag(R) >= 0.

Readings (the pages leave these open):
* Sigma goes into A' (eq. 4 keeps Sigma V^T as one matrix), so B' has
  orthonormal columns.  B' is stored transposed (k x d_out) next to A' (k x d_in).
* The factor-space route uses Delta W = Q_B (R_B R_A^T) Q_A^T, so the singular
  values of Delta W are those of the r x r matrix M = R_B R_A^T and its left
  singular vectors are Q_B U_M.
"""
from __future__ import annotations

import math

import numpy as np

F64 = np.float64


def qr_r(X) -> np.ndarray:
    """R factor of the thin QR of a tall matrix X (m x n, m >= n), diag(R) >= 0.

    The TSQR result (LoRAForge page, FlashTSQR section) written as its
    definition: a library Householder QR followed by the sign choice that makes
    R unique.
    """
    X = np.asarray(X, dtype=F64)
    R = np.linalg.qr(X, mode="r")
    d = np.sign(np.diag(R))
    d[d == 0] = 1.0
    return d[:, None] * R


def qr_q(X) -> np.ndarray:
    """Q factor of the same thin QR (columns orthonormal, sign-matched to qr_r)."""
    X = np.asarray(X, dtype=F64)
    Q, R = np.linalg.qr(X, mode="reduced")
    d = np.sign(np.diag(R))
    d[d == 0] = 1.0
    return Q * d[None, :]


def delta_w(B, A) -> np.ndarray:
    """Delta W = B A ("Compress then Serve" §3)."""
    return np.asarray(B, dtype=F64) @ np.asarray(A, dtype=F64)


def spectrum_dense(B, A):
    """Definition route: full SVD of the dense Delta W, truncated to r terms.

    Returns (sigma[r] descending, U d_out x r, Vt r x d_in).  Cost is that of
    a dense d_out x d_in SVD, so it is used on small and sampled modules.
    """
    r = np.asarray(B).shape[1]
    U, s, Vt = np.linalg.svd(delta_w(B, A), full_matrices=False)
    return s[:r].copy(), U[:, :r].copy(), Vt[:r].copy()


def spectrum_factor(B, A):
    """Factor-space route: R_B = R(B), R_A = R(A^T), M = R_B R_A^T, SVD(M).

    Returns (sigma[r] descending, U_M r x r, R_B, R_A).  sigma equals the
    singular values of Delta W and Q_B U_M its left singular vectors.
    """
    R_B = qr_r(B)
    R_A = qr_r(np.asarray(A, dtype=F64).T)
    M = R_B @ R_A.T
    U_M, s, _ = np.linalg.svd(M)
    return s, U_M, R_B, R_A


def export_dense(B, A, k: int):
    """Retained factors from the dense SVD: B'^T = U_k^T (k x d_out), A' = Sigma_k V_k^T."""
    s, U, Vt = spectrum_dense(B, A)
    return U[:, :k].T.copy(), s[:k, None] * Vt[:k]


def export_factor(B, A, k: int):
    """Retained factors from the factor-space route.

    B' = Q_B U_M[:, :k] (the top-k left singular vectors of Delta W) and
    A' = B'^T Delta W = U_M[:, :k]^T R_B A (= Sigma_k V_k^T).
    Returned as (B'^T k x d_out, A' k x d_in).
    """
    s, U_M, R_B, _ = spectrum_factor(B, A)
    Q_B = qr_q(B)
    Bp = Q_B @ U_M[:, :k]
    Ap = (U_M[:, :k].T @ R_B) @ np.asarray(A, dtype=F64)
    return Bp.T.copy(), Ap


def truncation_error(sigma, k: int) -> float:
    """Relative Frobenius error of the best rank-k approximation (Eckart-Young):
    sqrt(sum_{j>=k} sigma_j^2) / sqrt(sum_j sigma_j^2); 0 for a zero module."""
    s = np.asarray(sigma, dtype=F64)
    tot = math.fsum((s * s).tolist())
    if tot == 0.0:
        return 0.0
    tail = math.fsum((s[k:] * s[k:]).tolist())
    return math.sqrt(tail / tot)


def factor_error(B, A, Bt, Ap) -> float:
    """||B A - B' A'||_F / ||B A||_F for given retained factors, without forming
    any d_out x d_in matrix.

    Uses ||X - Y||^2 = ||X||^2 - 2<X, Y> + ||Y||^2 with
    ||B A||^2 = tr((B^T B)(A A^T)), <B A, B' A'> = tr((B'^T B)(A A'^T)),
    ||B' A'||^2 = tr((B'^T B')(A' A'^T)); every product is r x r, k x r or k x k.
    """
    B = np.asarray(B, dtype=F64); A = np.asarray(A, dtype=F64)
    Bt = np.asarray(Bt, dtype=F64); Ap = np.asarray(Ap, dtype=F64)
    xx = float(np.sum((B.T @ B) * (A @ A.T)))
    if xx == 0.0:
        return 0.0 if not np.any(Bt) or not np.any(Ap) else float("inf")
    xy = float(np.trace((Bt @ B) @ (A @ Ap.T)))
    yy = float(np.sum((Bt @ Bt.T) * (Ap @ Ap.T)))
    return math.sqrt(max(xx - 2.0 * xy + yy, 0.0) / xx)


def dense_error(B, A, Bt, Ap) -> float:
    """The same relative error computed densely (small modules only)."""
    X = delta_w(B, A)
    Y = np.asarray(Bt, dtype=F64).T @ np.asarray(Ap, dtype=F64)
    nx = np.linalg.norm(X)
    return 0.0 if nx == 0.0 else float(np.linalg.norm(X - Y) / nx)
