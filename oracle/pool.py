"""Pool-wide shared subspace of a LoRA pool, in float64 -- TEST INFRASTRUCTURE ONLY.

Source
------
* LoRASpace (the arXiv listing's abstract, "LoRASpace: A Pool-Wide Shared Substrate
  for Static and Dynamic Multi-LoRA Composition"): in real pools the stacked low-rank
  factors need far fewer directions than their summed ranks; the SVD of the stack gives
  the minimal subspace that keeps 99 % of the factor energy, computed once per pool and
  reused (reported as the retained fraction of the summed ranks, 46-57 % on diffusion
  pools).

Readings (the abstract gives no formula):
* "Stacked factors" of one module position: the row factors A_i (r_i x d_in) stacked
  as rows, S_A = [A_1; A_2; ...] (sum r_i x d_in), and the column factors B_i
  (d_out x r_i) side by side, S_B = [B_1 B_2 ...] (d_out x sum r_i).  Each side has
  its own subspace: the row space of S_A (directions in the input space) and the
  column space of S_B (directions in the output space).
* "Factor energy" is the squared Frobenius norm of the stack, sum_j sigma_j^2 over its
  singular values; "minimal subspace that keeps 99 %" is the smallest k with
  den * sum_{j<k} sigma_j^2 >= num * sum_j sigma_j^2 (num/den = 99/100), the same rule
  as the per-module energy fraction in ``allocate``, taken here with floor 1; the
  subspace is spanned by the k leading right (row stacks) or left (column stacks)
  singular vectors.
* The pools are used as given (no per-LoRA normalisation).

Nothing here is used by the CUDA path; the two share no code.
"""
from __future__ import annotations

import numpy as np

from .allocate import energy_fraction_rank


def stack_rows(As):
    """S_A = [A_1; A_2; ...]: the row factors (r_i x d) of a pool, stacked as rows."""
    As = [np.asarray(a, dtype=np.float64) for a in As]
    d = {a.shape[1] for a in As}
    if len(d) != 1:
        raise ValueError("row factors of one pool share their column count")
    return np.vstack(As)


def stack_cols(Bs):
    """S_B = [B_1 B_2 ...]: the column factors (d x r_i) of a pool, side by side."""
    Bs = [np.asarray(b, dtype=np.float64) for b in Bs]
    d = {b.shape[0] for b in Bs}
    if len(d) != 1:
        raise ValueError("column factors of one pool share their row count")
    return np.hstack(Bs)


def pool_subspace(factors, side: str = "row", num: int = 99, den: int = 100):
    """Minimal shared subspace of a pool's stacked factors (LoRASpace abstract).

    factors: the pool's A_i (side="row", each r_i x d) or B_i (side="col", each d x r_i).
    Returns dict(k, sigma, basis, frac, energy): k directions keep num/den of the
    stack's energy; sigma = singular values of the stack (descending); basis = d x k
    orthonormal (leading right singular vectors of S_A, or left ones of S_B);
    frac = k / sum r_i; energy = sum sigma^2."""
    if side == "row":
        S = stack_rows(factors)
        _, s, vt = np.linalg.svd(S, full_matrices=False)
        vecs = vt.T
    elif side == "col":
        S = stack_cols(factors)
        u, s, _ = np.linalg.svd(S, full_matrices=False)
        vecs = u
    else:
        raise ValueError("side is 'row' or 'col'")
    n = len(s)
    k, _ = energy_fraction_rank(s, n, num, den, 1)
    total_rank = sum((np.asarray(f).shape[0] if side == "row" else np.asarray(f).shape[1]) for f in factors)
    return dict(k=int(k), sigma=s, basis=vecs[:, :k], frac=k / total_rank, energy=float(np.sum(s * s)))


def project_pool(factors, basis, side: str = "row"):
    """Each LoRA's factor expressed in the shared basis (static reuse of the subspace):
    A_i ~= C_i basis^T with C_i = A_i basis (side="row"), or B_i ~= basis C_i with
    C_i = basis^T B_i (side="col").  Returns (coefficients, residual energy
    sum_i ||factor_i - reconstruction_i||_F^2)."""
    P = np.asarray(basis, dtype=np.float64)
    coefs, resid = [], 0.0
    for f in factors:
        f = np.asarray(f, dtype=np.float64)
        if side == "row":
            c = f @ P
            e = f - c @ P.T
        else:
            c = P.T @ f
            e = f - P @ c
        coefs.append(c)
        resid += float(np.sum(e * e))
    return coefs, resid
