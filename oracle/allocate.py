"""Retained-rank allocation: LoRAForge-U and LoRAForge-S, in float64.

Sources
-------
* LoRAForge abstract (mlinfo.pages.dev, arXiv 2611.01256): two policies share
  one backend -- uniform retention ratios (U) and spectral-energy budget
  allocation (S); the S "floored" configuration exports at 1/12 of rank with a
  rank floor.
* LoRAForge (kongchang.com), section "LoRAForge's Core Design: Explicit
  Retained-Rank Representation and Dual Strategies": U applies one retained
  ratio to every module; S allocates a total budget by each module's spectral
  energy accumulation curve, where spectral energy is the sum of squared
  singular values and each direction carries sigma_j^2 of it.

* LoRASpace (the arXiv listing's abstract, "LoRASpace: A Pool-Wide Shared Substrate
  for Static and Dynamic Multi-LoRA Composition"): the minimal subspace that keeps a
  fraction (99 %) of the factor energy, found by SVD.

Readings (the pages give no formula):
* U: k = round-half-up(num * r / den), clamped to [floor, r].
* S: budget in rank units per adapter (module ``group``):
  K = floor(num * sum_i r_i / den).  Every module first receives ``floor``.
  The remaining K - floor * M slots go to the candidates (i, j), j >= floor,
  with the largest normalised energy e_ij = sigma_ij^2 / sum_j sigma_ij^2
  (one module's accumulation curve, read per direction).  Candidates with
  e_ij = 0 are never taken, so budget can stay unused.  Equal energies are
  ordered by lower module index, then lower j.  Because e_ij does not increase
  with j, the chosen set is a prefix of every module, and the greedy choice
  maximises sum_i (retained energy fraction of module i) under sum_i k_i <= K.
  If K < floor * M every module keeps ``floor`` (budget exceeded, reported).
* Energy fraction (LoRASpace's rule read per module): k is the smallest rank in
  [floor, r] whose leading directions hold at least num/den of the module's
  spectral energy, den * sum_{j<k} sigma_j^2 >= num * sum_j sigma_j^2 (both sums
  taken in j order, ties keep the smaller k); a zero module keeps ``floor``.
"""
from __future__ import annotations

import math

import numpy as np


def uniform_rank(r: int, num: int, den: int, floor: int) -> int:
    """LoRAForge-U retained rank of a rank-r module."""
    k = (num * r + den // 2) // den
    return min(r, max(floor, k))


def energies(sigma, r: int, absolute: bool = False) -> np.ndarray:
    """Normalised spectral energies e_j = sigma_j^2 / sum sigma^2 (zeros for a zero
    module); with absolute=True the energies sigma_j^2 themselves."""
    s = np.asarray(sigma, dtype=np.float64)[:r]
    sq = s * s
    if absolute:
        return sq
    tot = math.fsum(sq.tolist())
    if tot == 0.0:
        return np.zeros(r)
    return sq / tot


def spectral_ranks(sigma_rows, r, group, num: int, den: int, floor: int, absolute: bool = False):
    """LoRAForge-S ranks for every module (absolute=True: the variant that ranks the
    candidates by sigma_ij^2, which minimises the group's summed squared Frobenius
    truncation error under the same budget).

    sigma_rows: n x r_max array, row i holds module i's singular values in
    descending order (entries past r_i ignored).
    Returns (ranks int32[n], info) where info[g] = dict(K, selected, gap_rel,
    over_budget) per group; gap_rel is the relative energy gap between the last
    selected and the first unselected candidate (inf if either does not exist).
    """
    sigma_rows = np.asarray(sigma_rows, dtype=np.float64)
    r = np.asarray(r); group = np.asarray(group)
    n = len(r)
    ranks = np.zeros(n, dtype=np.int32)
    info = {}
    for g in sorted(set(int(x) for x in group)):
        mods = [i for i in range(n) if int(group[i]) == g]
        K = (num * int(sum(int(r[i]) for i in mods))) // den
        extra = K - floor * len(mods)
        cands = []
        for i in mods:
            ri = int(r[i])
            if floor > ri:
                raise ValueError("floor exceeds module rank")
            if np.any(np.diff(sigma_rows[i][:ri]) > 0):
                raise ValueError("singular values must be listed in descending order")
            e = energies(sigma_rows[i], ri, absolute)
            for j in range(floor, ri):
                if e[j] > 0.0:
                    cands.append((-e[j], i, j))
        cands.sort()
        take = max(extra, 0)
        chosen = cands[:take]
        for i in mods:
            ranks[i] = floor
        for _, i, _ in chosen:
            ranks[i] += 1
        last = -chosen[-1][0] if chosen else None
        first_out = -cands[take][0] if take < len(cands) else None
        gap = math.inf
        if last is not None and first_out is not None and last > 0:
            gap = (last - first_out) / last
        info[g] = dict(K=K, selected=len(chosen), gap_rel=gap, over_budget=extra < 0)
    return ranks, info


def brute_force_ranks(sigma_rows, r, num: int, den: int, floor: int, absolute: bool = False):
    """Exhaustive search for one group (tiny cases only): every rank vector with
    floor <= k_i <= r_i and sum k_i <= K; returns (best objective, list of optimal
    rank tuples) for the objective sum_i sum_{j<k_i} e_ij."""
    import itertools
    sigma_rows = np.asarray(sigma_rows, dtype=np.float64)
    r = [int(x) for x in r]
    K = (num * sum(r)) // den
    E = [energies(sigma_rows[i], r[i], absolute) for i in range(len(r))]
    best, arg = -1.0, []
    for ks in itertools.product(*[range(floor, ri + 1) for ri in r]):
        if sum(ks) > max(K, floor * len(r)):
            continue
        val = math.fsum(math.fsum(E[i][:ks[i]].tolist()) for i in range(len(r)))
        tol = 1e-15 * max(abs(best), 1.0)
        if val > best + tol:
            best, arg = val, [ks]
        elif abs(val - best) <= tol:
            arg.append(ks)
    return best, arg


def energy_fraction_rank(sigma, r: int, num: int, den: int, floor: int):
    """Smallest k in [floor, r] with den * sum_{j<k} sigma_j^2 >= num * sum_j sigma_j^2.

    Returns (k, gap_rel): gap_rel = the smallest |den * cum_k - num * tot| / (num * tot)
    over k in [floor, r] (how far the module is from a tie at the threshold; inf for a
    zero module or num = 0)."""
    if floor > r:
        raise ValueError("floor exceeds module rank")
    s = np.asarray(sigma, dtype=np.float64)[:r]
    if np.any(np.diff(s) > 0):
        raise ValueError("singular values must be listed in descending order")
    sq = s * s
    tot = 0.0
    for v in sq:
        tot += float(v)
    if tot == 0.0:
        return floor, math.inf
    rhs = num * tot
    cum, k, gap = 0.0, None, math.inf
    for j in range(r):
        cum += float(sq[j])
        kk = j + 1
        if kk < floor:
            continue
        lhs = den * cum
        if rhs > 0.0:
            gap = min(gap, abs(lhs - rhs) / rhs)
        if k is None and lhs >= rhs:
            k = kk
    return (r if k is None else k), gap


def energy_fraction_ranks(sigma_rows, r, num: int, den: int, floor: int):
    """energy_fraction_rank for every module: (ranks int32[n], gaps float64[n])."""
    sigma_rows = np.asarray(sigma_rows, dtype=np.float64)
    out = [energy_fraction_rank(sigma_rows[i], int(r[i]), num, den, floor) for i in range(len(r))]
    return np.array([k for k, _ in out], dtype=np.int32), np.array([g for _, g in out])
